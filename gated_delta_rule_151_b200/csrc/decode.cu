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

// A lane's 16 columns of a row, or of k, q or a, are 8 column pairs: pair
// 2m holds columns 4(p + LPR m) + {0, 1}, pair 2m + 1 columns + {2, 3}, with
// p the lane's place in its row group.  The arithmetic runs on the packed
// fp32x2 units, two columns per instruction.
__device__ __forceinline__ void split4(float4 x, float2 &lo, float2 &hi) {
    lo = make_float2(x.x, x.y);
    hi = make_float2(x.z, x.w);
}

__device__ __forceinline__ float4 join4(float2 lo, float2 hi) {
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}

template <int LPR>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// kappa = k . q over the row group.
template <int LPR>
__device__ __forceinline__ float head_kappa(const float2 (&k)[8], const float2 (&q)[8]) {
    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 8; ++j) acc = __ffma2_rn(k[j], q[j], acc);
    return group_sum<LPR>(acc.x + acc.y);
}

// One token applied to one state row (the lane's 16 columns in e); returns
// o_r.  Every decode kernel goes through this routine, so several tokens in
// one pass give bit for bit the results of as many single steps.
template <int LPR, bool CHANNEL>
__device__ __forceinline__ float row_token(float2 (&e)[8], const float2 (&k)[8],
                                           const float2 (&q)[8],
                                           const float2 (&a)[CHANNEL ? 8 : 1], float b, float vr,
                                           float kappa) {
    float2 x2 = make_float2(0.f, 0.f), y2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        e[j] = __fmul2_rn(e[j], CHANNEL ? a[j] : a[0]);
        x2 = __ffma2_rn(e[j], k[j], x2);
        y2 = __ffma2_rn(e[j], q[j], y2);
    }
    const float x = group_sum<LPR>(x2.x + x2.y);
    const float y = group_sum<LPR>(y2.x + y2.y);
    const float u = b * (vr - x);
    const float2 u2 = make_float2(u, u);
#pragma unroll
    for (int j = 0; j < 8; ++j) e[j] = __ffma2_rn(u2, k[j], e[j]);
    return fmaf(u, kappa, y);
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
    float2 s[MAXP][8];
#pragma unroll
    for (int pp = 0; pp < MAXP; ++pp) {
        const int r = pp * RP + rg;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float4 x = (r < DV) ? __ldcs(S + (size_t)r * (DK / 4) + p + LPR * m)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
            split4(x, s[pp][2 * m], s[pp][2 * m + 1]);
        }
    }

    float2 kf[8], qf[8], af[CHANNEL ? 8 : 1];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int col = 4 * (p + LPR * m);
        float t[4];
        load4(k + qh * DK + col, t);
        kf[2 * m] = make_float2(t[0], t[1]);
        kf[2 * m + 1] = make_float2(t[2], t[3]);
        load4(q + qh * DK + col, t);
        qf[2 * m] = make_float2(t[0], t[1]);
        qf[2 * m + 1] = make_float2(t[2], t[3]);
    }
    if constexpr (CHANNEL) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int col = 4 * (p + LPR * m);
            const float4 gg = *reinterpret_cast<const float4 *>(g + nh * DK + col);
            af[2 * m] = make_float2(__expf(clamp_log_gate(gg.x)), __expf(clamp_log_gate(gg.y)));
            af[2 * m + 1] = make_float2(__expf(clamp_log_gate(gg.z)), __expf(clamp_log_gate(gg.w)));
        }
    } else {
        const float a = __expf(clamp_log_gate(g[nh]));
        af[0] = make_float2(a, a);
    }
    const float b = beta[nh];
    const float kappa = head_kappa<LPR>(kf, qf);

#pragma unroll
    for (int pp = 0; pp < MAXP; ++pp) {
        const int r = pp * RP + rg;
        const float vr = (r < DV) ? to_f32(v[nh * DV + r]) : 0.f;
        const float out = row_token<LPR, CHANNEL>(s[pp], kf, qf, af, b, vr, kappa);
        if (r < DV) {
#pragma unroll
            for (int m = 0; m < 4; ++m)
                __stcs(S + (size_t)r * (DK / 4) + p + LPR * m, join4(s[pp][2 * m], s[pp][2 * m + 1]));
            if (p == 0) store_io(o + nh * DV + r, out);
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
// written once, so the state traffic per token falls by T.  Optionally the
// state after every token is stored to a snapshot buffer, from which a
// caller rolls back to the last accepted draft token.
//
// With T updates per row the arithmetic is no longer small next to the
// bytes, so the kernel overlaps the two: it is persistent, and each CTA walks
// over slabs of RB state rows of one (sequence, head) -- RB * d_k * 4
// contiguous bytes -- with a ring of kMultiStages shared-memory stages that
// cp.async fills kMultiStages - 1 slabs ahead.  A stage holds the slab's
// state rows and the T tokens' k, q, the slab's v entries, the gates and
// beta.  Data in flight costs no registers, so a few CTAs per SM keep the
// HBM pipe full while the arithmetic of the current slab runs.  Two stages
// (one slab ahead) leave room for three CTAs per SM at d = 128, T = 4; on
// B200 that beat three stages at two CTAs per SM by 18 %, because the
// per-token row updates are latency-bound and want the extra warps.
constexpr int kMultiThreads = 128;
constexpr int kMultiStages = 2;

template <int DK>
struct MultiShape {
    static constexpr int LPR = DK / 16;                       // lanes per row
    static constexpr int RP = kMultiThreads / LPR;            // rows per pass
    static constexpr int MAXP = (LPR / 2 > 0) ? LPR / 2 : 1;  // passes per slab
    static constexpr int RB = RP * MAXP;                      // rows per slab
};

__host__ __device__ constexpr int align16(int x) { return (x + 15) & ~15; }

// Byte offsets inside a stage, the stage stride, and the fp32 operand
// buffer (k, q converted once per slab; exp of the gates) after the ring.
struct MultiLayout {
    int st, kq, v, g, b, stage, conv_kq, conv_a, total;
};

__host__ __device__ inline MultiLayout multi_layout(int T, int DK, int RB, int io_bytes, int GD) {
    MultiLayout L;
    L.st = 0;
    L.kq = RB * DK * 4;
    L.v = L.kq + align16(T * 2 * DK * io_bytes);
    L.g = L.v + align16(T * RB * io_bytes);
    L.b = L.g + align16(T * GD * 4);
    L.stage = (L.b + T * 4 + 127) & ~127;
    L.conv_kq = kMultiStages * L.stage;
    L.conv_a = L.conv_kq + T * 2 * DK * 4;
    L.total = L.conv_a + align16(T * GD * 4);
    return L;
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}

__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Slab s = (sequence, head) * nblk + row block.
struct Slab {
    size_t nh, n;
    int h, r0, rows;
};

__device__ __forceinline__ Slab slab_of(long long s, int nblk, int H, int RB, int DV) {
    Slab x;
    x.nh = (size_t)(s / nblk);
    x.r0 = (int)(s % nblk) * RB;
    x.n = x.nh / H;
    x.h = (int)(x.nh % H);
    x.rows = min(RB, DV - x.r0);
    return x;
}

// Start the copies of one slab into a stage (every thread takes a share).
// All sources are 16-byte aligned (the C ABI checks the base pointers; rows
// are multiples of 16 elements), except scalar gates and beta: 4-byte copies.
template <int DK, bool CHANNEL, typename IoT>
__device__ __forceinline__ void issue_slab(uint8_t *stg, const MultiLayout &L, const Slab &x,
                                           const IoT *q, const IoT *k, const IoT *v,
                                           const float *g, const float *beta, const float *state,
                                           int T, int Hqk, int H, int DV) {
    constexpr int RB = MultiShape<DK>::RB;
    const int tid = threadIdx.x;
    const size_t hq = (size_t)(x.h / (H / Hqk));
    const float *src = state + (x.nh * DV + x.r0) * DK;
    const int ns = x.rows * DK / 4;
    for (int i = tid; i < ns; i += kMultiThreads) cp_async16(stg + L.st + 16 * i, src + 4 * i);
    constexpr int KG = DK * (int)sizeof(IoT) / 16;     // 16-byte pieces of a k or q row
    for (int i = tid; i < T * 2 * KG; i += kMultiThreads) {
        const int t = i / (2 * KG), w = (i / KG) % 2, c = i % KG;
        const IoT *row = (w == 0 ? k : q) + ((x.n * T + t) * Hqk + hq) * DK;
        cp_async16(stg + L.kq + (2 * t + w) * DK * (int)sizeof(IoT) + 16 * c,
                   reinterpret_cast<const uint8_t *>(row) + 16 * c);
    }
    const int VG = x.rows * (int)sizeof(IoT) / 16;
    for (int i = tid; i < T * VG; i += kMultiThreads) {
        const int t = i / VG, c = i % VG;
        const IoT *row = v + ((x.n * T + t) * H + x.h) * DV + x.r0;
        cp_async16(stg + L.v + t * RB * (int)sizeof(IoT) + 16 * c,
                   reinterpret_cast<const uint8_t *>(row) + 16 * c);
    }
    if constexpr (CHANNEL) {
        for (int i = tid; i < T * (DK / 4); i += kMultiThreads) {
            const int t = i / (DK / 4), c = i % (DK / 4);
            cp_async16(stg + L.g + (t * DK + 4 * c) * 4, g + ((x.n * T + t) * H + x.h) * DK + 4 * c);
        }
    } else {
        for (int t = tid; t < T; t += kMultiThreads)
            cp_async4(stg + L.g + 4 * t, g + (x.n * T + t) * H + x.h);
    }
    for (int t = tid; t < T; t += kMultiThreads)
        cp_async4(stg + L.b + 4 * t, beta + (x.n * T + t) * H + x.h);
}

template <int DK, bool CHANNEL, typename IoT>
__global__ void __launch_bounds__(kMultiThreads, 3)
decode_multi_kernel(const IoT *__restrict__ q, const IoT *__restrict__ k,
                    const IoT *__restrict__ v, const float *__restrict__ g,
                    const float *__restrict__ beta, float *__restrict__ state, int T, int Hqk,
                    int H, int DV, int nblk, long long slabs, IoT *__restrict__ o,
                    float *__restrict__ snap) {
    using Sh = MultiShape<DK>;
    constexpr int LPR = Sh::LPR, RP = Sh::RP, MAXP = Sh::MAXP, RB = Sh::RB;
    constexpr int GD = CHANNEL ? DK : 1;
    extern __shared__ __align__(128) uint8_t smem[];
    const MultiLayout L = multi_layout(T, DK, RB, (int)sizeof(IoT), GD);
    const int tid = threadIdx.x;
    const int p = tid % LPR;
    const int rg = tid / LPR;
    const long long first = blockIdx.x, stride = gridDim.x;
    const int mine = slabs > first ? (int)((slabs - 1 - first) / stride + 1) : 0;
    float *kqf = reinterpret_cast<float *>(smem + L.conv_kq);   // [T][2][DK]  k, q
    float *af = reinterpret_cast<float *>(smem + L.conv_a);     // [T][GD]     exp(g)

#pragma unroll
    for (int j = 0; j < kMultiStages - 1; ++j) {
        if (j < mine)
            issue_slab<DK, CHANNEL, IoT>(smem + j * L.stage, L,
                                         slab_of(first + j * stride, nblk, H, RB, DV), q, k, v,
                                         g, beta, state, T, Hqk, H, DV);
        cp_async_commit();
    }

    for (int j = 0; j < mine; ++j) {
        const int jn = j + kMultiStages - 1;
        if (jn < mine)
            issue_slab<DK, CHANNEL, IoT>(smem + (jn % kMultiStages) * L.stage, L,
                                         slab_of(first + jn * stride, nblk, H, RB, DV), q, k, v,
                                         g, beta, state, T, Hqk, H, DV);
        cp_async_commit();
        cp_async_wait<kMultiStages - 1>();   // slab j has landed (groups complete in order)
        __syncthreads();

        const uint8_t *stg = smem + (j % kMultiStages) * L.stage;
        const Slab x = slab_of(first + j * stride, nblk, H, RB, DV);
        const IoT *kq_raw = reinterpret_cast<const IoT *>(stg + L.kq);
        for (int i = tid; i < T * 2 * DK; i += kMultiThreads) kqf[i] = to_f32(kq_raw[i]);
        const float *g_raw = reinterpret_cast<const float *>(stg + L.g);
        for (int i = tid; i < T * GD; i += kMultiThreads) af[i] = __expf(clamp_log_gate(g_raw[i]));

        const float4 *st4 = reinterpret_cast<const float4 *>(stg + L.st);
        float2 s[MAXP][8];
#pragma unroll
        for (int pp = 0; pp < MAXP; ++pp) {
            const int rl = pp * RP + rg;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 e4 = (rl < x.rows) ? st4[rl * (DK / 4) + p + LPR * m]
                                                : make_float4(0.f, 0.f, 0.f, 0.f);
                split4(e4, s[pp][2 * m], s[pp][2 * m + 1]);
            }
        }
        __syncthreads();   // converted operands visible

        const IoT *v_raw = reinterpret_cast<const IoT *>(stg + L.v);
        const float *b_raw = reinterpret_cast<const float *>(stg + L.b);
        for (int t = 0; t < T; ++t) {
            float2 kf[8], qf[8], a2[CHANNEL ? 8 : 1];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int col = 4 * (p + LPR * m);
                split4(*reinterpret_cast<const float4 *>(kqf + (2 * t) * DK + col), kf[2 * m],
                       kf[2 * m + 1]);
                split4(*reinterpret_cast<const float4 *>(kqf + (2 * t + 1) * DK + col), qf[2 * m],
                       qf[2 * m + 1]);
                if constexpr (CHANNEL)
                    split4(*reinterpret_cast<const float4 *>(af + t * DK + col), a2[2 * m],
                           a2[2 * m + 1]);
            }
            if constexpr (!CHANNEL) a2[0] = make_float2(af[t], af[t]);
            const float b = b_raw[t];
            const float kappa = head_kappa<LPR>(kf, qf);
            // every row first (their dependency chains interleave), then the stores
            float out[MAXP];
#pragma unroll
            for (int pp = 0; pp < MAXP; ++pp) {
                const int rl = pp * RP + rg;
                const float vr = (rl < x.rows) ? to_f32(v_raw[t * RB + rl]) : 0.f;
                out[pp] = row_token<LPR, CHANNEL>(s[pp], kf, qf, a2, b, vr, kappa);
            }
            const size_t vrow = (x.n * T + t) * H + x.h;
#pragma unroll
            for (int pp = 0; pp < MAXP; ++pp) {
                const int rl = pp * RP + rg;
                if (rl < x.rows) {
                    const int r = x.r0 + rl;
                    if (snap != nullptr) {
#pragma unroll
                        for (int m = 0; m < 4; ++m)
                            __stcs(reinterpret_cast<float4 *>(snap + (vrow * DV + r) * DK) + p + LPR * m,
                                   join4(s[pp][2 * m], s[pp][2 * m + 1]));
                    }
                    if (p == 0) store_io(o + vrow * DV + r, out[pp]);
                }
            }
        }
        float4 *S = reinterpret_cast<float4 *>(state + (x.nh * DV + x.r0) * DK);
#pragma unroll
        for (int pp = 0; pp < MAXP; ++pp) {
            const int rl = pp * RP + rg;
            if (rl < x.rows) {
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    __stcs(S + (size_t)rl * (DK / 4) + p + LPR * m, join4(s[pp][2 * m], s[pp][2 * m + 1]));
            }
        }
        __syncthreads();   // the stage and the operand buffer are free again
    }
    cp_async_wait<0>();
}

// CTAs per SM the multi-token kernel reaches with a given shared memory
// size (cached: the occupancy query costs host time on every launch).
inline cudaError_t resident_ctas(const void *fn, int threads, int smem, int *out) {
    struct Entry {
        const void *fn;
        int dev, smem, ctas;
    };
    static std::mutex mu;
    static std::vector<Entry> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    for (auto &d : done)
        if (d.fn == fn && d.dev == dev && d.smem == smem) {
            *out = d.ctas;
            return cudaSuccess;
        }
    int sms = 0, per = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, fn, threads, smem);
    if (e != cudaSuccess) return e;
    if (per < 1) return cudaErrorInvalidConfiguration;
    done.push_back(Entry{fn, dev, smem, sms * per});
    *out = sms * per;
    return cudaSuccess;
}

template <int DK, bool CHANNEL, typename IoT>
cudaError_t launch_multi_dk(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, float *state, int N, int T, int Hqk, int H, int DV,
                            void *o, float *snap, cudaStream_t stream) {
    using Sh = MultiShape<DK>;
    const MultiLayout L = multi_layout(T, DK, Sh::RB, (int)sizeof(IoT), CHANNEL ? DK : 1);
    auto kern = decode_multi_kernel<DK, CHANNEL, IoT>;
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void *>(kern), L.total);
    if (e != cudaSuccess) return e;
    int ctas = 0;
    e = resident_ctas(reinterpret_cast<const void *>(kern), kMultiThreads, L.total, &ctas);
    if (e != cudaSuccess) return e;
    const int nblk = (DV + Sh::RB - 1) / Sh::RB;
    const long long slabs = (long long)N * H * nblk;
    const unsigned grid = (unsigned)(slabs < ctas ? slabs : ctas);
    kern<<<grid, kMultiThreads, L.total, stream>>>(
        static_cast<const IoT *>(q), static_cast<const IoT *>(k), static_cast<const IoT *>(v), g,
        beta, state, T, Hqk, H, DV, nblk, slabs, static_cast<IoT *>(o), snap);
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
