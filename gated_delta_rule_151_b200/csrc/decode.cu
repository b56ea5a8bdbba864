// Single-token decode step of the gated delta rule.
//
// For one new token per (sequence n, head h) the state update of the page
// "How the New Flash Models Work: Inside GLM-5.3-Flash and Qwen3.8-Flash-Next"
// (section "Linear attention: a fixed-size memory in place of the cache",
// Gated DeltaNet and Kimi Delta Attention equations) acts on every row r of
// S (value channel r) independently:
//
//     s_r  = S_r ⊙ a                  (a = exp(g): scalar, or one per key channel)
//     x_r  = s_r · k,   y_r = s_r · q
//     u_r  = beta (v_r - x_r)
//     S_r <- s_r + u_r k
//     o_r  = S_r · q = y_r + u_r (k · q)
//
// so the whole step is one read-modify-write pass over the fp32 state, which
// makes it HBM-bound (the pages describe decode as bound by memory
// bandwidth).  Layout: a row is d_k contiguous fp32; LPR = d_k / 16 lanes
// share a row, each holding 16 columns as four float4 spread so that, for
// each of the four loads, the LPR lanes of a row read LPR*16 consecutive
// bytes.  A 256-thread block owns one (n, h) pair and issues every one of its
// row loads before any arithmetic, so each thread keeps up to 256 bytes of
// state in flight.  The dot products are finished with xor shuffles inside
// the row's lane group.  State loads and stores use the streaming
// (evict-first) cache hints: the state is touched once per step.
#include "common.cuh"

namespace gdr {
namespace {

constexpr int kDecodeThreads = 256;

__device__ __forceinline__ void load4(const float *p, float out[4]) {
    float4 x = *reinterpret_cast<const float4 *>(p);
    out[0] = x.x; out[1] = x.y; out[2] = x.z; out[3] = x.w;
}

__device__ __forceinline__ void load4(const __nv_bfloat16 *p, float out[4]) {
    uint2 raw = *reinterpret_cast<const uint2 *>(p);
    __nv_bfloat162 lo = *reinterpret_cast<__nv_bfloat162 *>(&raw.x);
    __nv_bfloat162 hi = *reinterpret_cast<__nv_bfloat162 *>(&raw.y);
    float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
    out[0] = a.x; out[1] = a.y; out[2] = b.x; out[3] = b.y;
}

template <int DK, bool CHANNEL, typename IoT>
__global__ void __launch_bounds__(kDecodeThreads, 2)
decode_step_kernel(const IoT *__restrict__ q, const IoT *__restrict__ k,
                   const IoT *__restrict__ v, const float *__restrict__ g,
                   const float *__restrict__ beta, float *__restrict__ state, int Hqk, int H,
                   int DV, IoT *__restrict__ o) {
    constexpr int LPR = DK / 16;                      // lanes per state row
    constexpr int RP = kDecodeThreads / LPR;          // rows per pass
    constexpr int MAXP = (LPR / 2 > 0) ? LPR / 2 : 1; // passes cover d_v <= 128
    static_assert(MAXP * RP >= 128, "passes must cover 128 rows");

    const size_t nh = blockIdx.x;                       // (sequence, value head)
    const size_t qh = (nh / H) * Hqk + (nh % H) / (H / Hqk);   // its query/key head
    const int tid = threadIdx.x;
    const int p = tid % LPR;
    const int rg = tid / LPR;

    float4 *S = reinterpret_cast<float4 *>(state + nh * (size_t)DV * DK);

    // Issue all state loads of this thread first.
    float4 s[MAXP][4];
#pragma unroll
    for (int pp = 0; pp < MAXP; ++pp) {
        const int r = pp * RP + rg;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            if (r < DV)
                s[pp][m] = __ldcs(S + (size_t)r * (DK / 4) + p + LPR * m);
            else
                s[pp][m] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }

    float kf[16], qf[16];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int col = 4 * (p + LPR * m);
        load4(k + qh * DK + col, kf + 4 * m);
        load4(q + qh * DK + col, qf + 4 * m);
    }
    float af[CHANNEL ? 16 : 1];
    if constexpr (CHANNEL) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int col = 4 * (p + LPR * m);
            float4 gg = *reinterpret_cast<const float4 *>(g + nh * DK + col);
            af[4 * m + 0] = __expf(clamp_log_gate(gg.x));
            af[4 * m + 1] = __expf(clamp_log_gate(gg.y));
            af[4 * m + 2] = __expf(clamp_log_gate(gg.z));
            af[4 * m + 3] = __expf(clamp_log_gate(gg.w));
        }
    } else {
        af[0] = __expf(clamp_log_gate(g[nh]));
    }
    const float b = beta[nh];

    // kappa = k . q, shared by every row of the head.
    float kappa = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) kappa = fmaf(kf[i], qf[i], kappa);
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) kappa += __shfl_xor_sync(0xffffffffu, kappa, off);

#pragma unroll
    for (int pp = 0; pp < MAXP; ++pp) {
        const int r = pp * RP + rg;
        float x = 0.f, y = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            float *e = reinterpret_cast<float *>(&s[pp][m]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float a = CHANNEL ? af[4 * m + c] : af[0];
                e[c] *= a;
                x = fmaf(e[c], kf[4 * m + c], x);
                y = fmaf(e[c], qf[4 * m + c], y);
            }
        }
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) {
            x += __shfl_xor_sync(0xffffffffu, x, off);
            y += __shfl_xor_sync(0xffffffffu, y, off);
        }
        if (r < DV) {
            const float u = b * (to_f32(v[nh * DV + r]) - x);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                float *e = reinterpret_cast<float *>(&s[pp][m]);
#pragma unroll
                for (int c = 0; c < 4; ++c) e[c] = fmaf(u, kf[4 * m + c], e[c]);
                __stcs(S + (size_t)r * (DK / 4) + p + LPR * m, s[pp][m]);
            }
            if (p == 0) store_io(o + nh * DV + r, fmaf(u, kappa, y));
        }
    }
}

template <int DK, bool CHANNEL, typename IoT>
cudaError_t launch_dk(const void *q, const void *k, const void *v, const float *g,
                      const float *beta, float *state, int N, int Hqk, int H, int DV, void *o,
                      cudaStream_t stream) {
    const unsigned blocks = (unsigned)((size_t)N * H);
    decode_step_kernel<DK, CHANNEL, IoT><<<blocks, kDecodeThreads, 0, stream>>>(
        static_cast<const IoT *>(q), static_cast<const IoT *>(k), static_cast<const IoT *>(v), g,
        beta, state, Hqk, H, DV, static_cast<IoT *>(o));
    return cudaGetLastError();
}

template <bool CHANNEL, typename IoT>
cudaError_t launch_mode(const void *q, const void *k, const void *v, const float *g,
                        const float *beta, float *state, int N, int Hqk, int H, int DK,
                        int DV, void *o, cudaStream_t stream) {
    switch (DK) {
        case 16: return launch_dk<16, CHANNEL, IoT>(q, k, v, g, beta, state, N, Hqk, H, DV, o, stream);
        case 32: return launch_dk<32, CHANNEL, IoT>(q, k, v, g, beta, state, N, Hqk, H, DV, o, stream);
        case 64: return launch_dk<64, CHANNEL, IoT>(q, k, v, g, beta, state, N, Hqk, H, DV, o, stream);
        default: return launch_dk<128, CHANNEL, IoT>(q, k, v, g, beta, state, N, Hqk, H, DV, o, stream);
    }
}

// ------------------------------------------------------ several tokens ----
//
// T consecutive tokens of each sequence in one pass over the state (draft
// verification in speculative decoding): every state row is read once, the
// T updates are applied in registers token after token, and the row is
// written once, so the state traffic per token falls by T.  The T tokens'
// q/k/v/gates/beta of the (sequence, head) are staged in shared memory while
// the state loads are in flight.  Optionally the state after every token is
// stored to a snapshot buffer, from which a caller rolls back to the last
// accepted draft token.
template <int DK, bool CHANNEL, typename IoT>
__global__ void __launch_bounds__(kDecodeThreads, 2)
decode_multi_kernel(const IoT *__restrict__ q, const IoT *__restrict__ k,
                    const IoT *__restrict__ v, const float *__restrict__ g,
                    const float *__restrict__ beta, float *__restrict__ state, int T, int Hqk,
                    int H, int DV, IoT *__restrict__ o, float *__restrict__ snap) {
    constexpr int LPR = DK / 16;
    constexpr int RP = kDecodeThreads / LPR;
    constexpr int MAXP = (LPR / 2 > 0) ? LPR / 2 : 1;
    constexpr int GD = CHANNEL ? DK : 1;
    extern __shared__ float sh[];

    const size_t nh = blockIdx.x;                 // (sequence, value head)
    const size_t n = nh / H, h = nh % H;
    const size_t hq = h / (H / Hqk);
    const int tid = threadIdx.x;
    const int p = tid % LPR;
    const int rg = tid / LPR;

    float4 *S = reinterpret_cast<float4 *>(state + nh * (size_t)DV * DK);
    float4 s[MAXP][4];
#pragma unroll
    for (int pp = 0; pp < MAXP; ++pp) {
        const int r = pp * RP + rg;
#pragma unroll
        for (int m = 0; m < 4; ++m)
            s[pp][m] = (r < DV) ? __ldcs(S + (size_t)r * (DK / 4) + p + LPR * m)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
    }

    float *kq = sh;                       // [T][2][DK]  k, q
    float *vs = kq + (size_t)T * 2 * DK;  // [T][DV]
    float *as = vs + (size_t)T * DV;      // [T][GD]     exp(g)
    float *bs = as + (size_t)T * GD;      // [T]
    for (int idx = tid; idx < T * DK; idx += kDecodeThreads) {
        const int t = idx / DK, c = idx % DK;
        const size_t qrow = (n * T + t) * Hqk + hq;
        kq[(2 * t) * DK + c] = to_f32(k[qrow * DK + c]);
        kq[(2 * t + 1) * DK + c] = to_f32(q[qrow * DK + c]);
    }
    for (int idx = tid; idx < T * DV; idx += kDecodeThreads) {
        const int t = idx / DV, r = idx % DV;
        vs[idx] = to_f32(v[((n * T + t) * H + h) * DV + r]);
    }
    for (int idx = tid; idx < T * GD; idx += kDecodeThreads) {
        const int t = idx / GD, c = idx % GD;
        as[idx] = __expf(clamp_log_gate(g[((n * T + t) * H + h) * GD + c]));
    }
    for (int t = tid; t < T; t += kDecodeThreads) bs[t] = beta[(n * T + t) * H + h];
    __syncthreads();

    for (int t = 0; t < T; ++t) {
        float kf[16], qf[16], af[CHANNEL ? 16 : 1];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int col = 4 * (p + LPR * m);
            const float4 kk = *reinterpret_cast<const float4 *>(kq + (2 * t) * DK + col);
            const float4 qq = *reinterpret_cast<const float4 *>(kq + (2 * t + 1) * DK + col);
            kf[4 * m] = kk.x; kf[4 * m + 1] = kk.y; kf[4 * m + 2] = kk.z; kf[4 * m + 3] = kk.w;
            qf[4 * m] = qq.x; qf[4 * m + 1] = qq.y; qf[4 * m + 2] = qq.z; qf[4 * m + 3] = qq.w;
            if constexpr (CHANNEL) {
                const float4 aa = *reinterpret_cast<const float4 *>(as + t * DK + col);
                af[4 * m] = aa.x; af[4 * m + 1] = aa.y; af[4 * m + 2] = aa.z; af[4 * m + 3] = aa.w;
            }
        }
        if constexpr (!CHANNEL) af[0] = as[t];
        const float b = bs[t];
        float kappa = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) kappa = fmaf(kf[i], qf[i], kappa);
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) kappa += __shfl_xor_sync(0xffffffffu, kappa, off);

        const size_t vrow = (n * T + t) * H + h;
#pragma unroll
        for (int pp = 0; pp < MAXP; ++pp) {
            const int r = pp * RP + rg;
            float x = 0.f, y = 0.f;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                float *e = reinterpret_cast<float *>(&s[pp][m]);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    e[c] *= CHANNEL ? af[4 * m + c] : af[0];
                    x = fmaf(e[c], kf[4 * m + c], x);
                    y = fmaf(e[c], qf[4 * m + c], y);
                }
            }
#pragma unroll
            for (int off = LPR / 2; off > 0; off >>= 1) {
                x += __shfl_xor_sync(0xffffffffu, x, off);
                y += __shfl_xor_sync(0xffffffffu, y, off);
            }
            if (r < DV) {
                const float u = b * (vs[t * DV + r] - x);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    float *e = reinterpret_cast<float *>(&s[pp][m]);
#pragma unroll
                    for (int c = 0; c < 4; ++c) e[c] = fmaf(u, kf[4 * m + c], e[c]);
                    if (snap != nullptr)
                        __stcs(reinterpret_cast<float4 *>(snap + (vrow * DV + r) * DK) + p + LPR * m,
                               s[pp][m]);
                }
                if (p == 0) store_io(o + vrow * DV + r, fmaf(u, kappa, y));
            }
        }
    }
#pragma unroll
    for (int pp = 0; pp < MAXP; ++pp) {
        const int r = pp * RP + rg;
        if (r < DV) {
#pragma unroll
            for (int m = 0; m < 4; ++m) __stcs(S + (size_t)r * (DK / 4) + p + LPR * m, s[pp][m]);
        }
    }
}

template <int DK, bool CHANNEL, typename IoT>
cudaError_t launch_multi_dk(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, float *state, int N, int T, int Hqk, int H, int DV,
                            void *o, float *snap, cudaStream_t stream) {
    const size_t smem = sizeof(float) * (size_t)T * (2 * DK + DV + (CHANNEL ? DK : 1) + 1);
    auto kern = decode_multi_kernel<DK, CHANNEL, IoT>;
    if (smem > 48 * 1024) {
        cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void *>(kern), (int)smem);
        if (e != cudaSuccess) return e;
    }
    const unsigned blocks = (unsigned)((size_t)N * H);
    kern<<<blocks, kDecodeThreads, smem, stream>>>(
        static_cast<const IoT *>(q), static_cast<const IoT *>(k), static_cast<const IoT *>(v), g,
        beta, state, T, Hqk, H, DV, static_cast<IoT *>(o), snap);
    return cudaGetLastError();
}

template <bool CHANNEL, typename IoT>
cudaError_t launch_multi_mode(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, float *state, int N, int T, int Hqk, int H,
                              int DK, int DV, void *o, float *snap, cudaStream_t stream) {
    switch (DK) {
        case 16: return launch_multi_dk<16, CHANNEL, IoT>(q, k, v, g, beta, state, N, T, Hqk, H, DV, o, snap, stream);
        case 32: return launch_multi_dk<32, CHANNEL, IoT>(q, k, v, g, beta, state, N, T, Hqk, H, DV, o, snap, stream);
        case 64: return launch_multi_dk<64, CHANNEL, IoT>(q, k, v, g, beta, state, N, T, Hqk, H, DV, o, snap, stream);
        default: return launch_multi_dk<128, CHANNEL, IoT>(q, k, v, g, beta, state, N, T, Hqk, H, DV, o, snap, stream);
    }
}

}  // namespace

// Host launcher (arguments already validated by the C ABI layer).
cudaError_t launch_decode_step(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, float *state, int N, int Hqk, int H, int DK,
                               int DV, bool channel, bool bf16, void *o, cudaStream_t stream) {
    if (N == 0 || H == 0) return cudaSuccess;
    if (channel)
        return bf16 ? launch_mode<true, __nv_bfloat16>(q, k, v, g, beta, state, N, Hqk, H, DK, DV, o, stream)
                    : launch_mode<true, float>(q, k, v, g, beta, state, N, Hqk, H, DK, DV, o, stream);
    return bf16 ? launch_mode<false, __nv_bfloat16>(q, k, v, g, beta, state, N, Hqk, H, DK, DV, o, stream)
                : launch_mode<false, float>(q, k, v, g, beta, state, N, Hqk, H, DK, DV, o, stream);
}

}  // namespace gdr

namespace gdr {

cudaError_t launch_decode_multi(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, float *state, int N, int T, int Hqk, int H,
                                int DK, int DV, bool channel, bool bf16, void *o, float *snap,
                                cudaStream_t stream) {
    if (N == 0 || H == 0 || T == 0) return cudaSuccess;
    if (channel)
        return bf16 ? launch_multi_mode<true, __nv_bfloat16>(q, k, v, g, beta, state, N, T, Hqk, H, DK, DV, o, snap, stream)
                    : launch_multi_mode<true, float>(q, k, v, g, beta, state, N, T, Hqk, H, DK, DV, o, snap, stream);
    return bf16 ? launch_multi_mode<false, __nv_bfloat16>(q, k, v, g, beta, state, N, T, Hqk, H, DK, DV, o, snap, stream)
                : launch_multi_mode<false, float>(q, k, v, g, beta, state, N, T, Hqk, H, DK, DV, o, snap, stream);
}

}  // namespace gdr
