// Gradient of the gated delta-rule recurrence (the rule of the page "How the
// New Flash Models Work: Inside GLM-5.3-Flash and Qwen3.8-Flash-Next",
// section "Linear attention: a fixed-size memory in place of the cache"; the
// pages train these layers but print no backward pass).
//
// Per row r of the state (value channel r), with a_t = exp(g_t):
//
//     e = s_{t-1} * a_t,  x = e . k_t,  u = beta_t (v_r - x),  s_t = e + u k_t,
//     o_r = s_t . q_t
//
// and for the loss <dO, O> + <dS_final, S_final> the adjoint ds of s_t runs
// backwards, row by row as well:
//
//     ds += dO_r q_t;          dq_t += dO_r s_t
//     du = ds . k_t;           dk_t += u ds + dx e,   dx = -beta_t du
//     dbeta_t += (v_r - x) du; dv_r = beta_t du
//     dE = ds + dx k_t;        dg_t += (dE * s_{t-1}) a_t   (summed over
//                                  columns too for the scalar gate)
//     ds = dE * a_t
//
// Rows are independent in both directions, so a CTA owns a block of RB rows
// of one (sequence, head): the d_k / 16 lanes of a row hold 16 columns each,
// as in the decode kernel.  Only the sums over rows (dq, dk, dg, dbeta) cross
// CTAs.  Per token every thread writes its row's parts to shared memory and,
// after a barrier, each column is summed over the CTA's rows by one thread
// (no shared-memory atomics); the chunk's sums are then added to the
// zero-filled outputs with global atomics.
//
// Two sweeps.  The forward sweep runs the recurrence and writes the state
// before every chunk of kBwdChunk tokens to the workspace.  The reverse sweep
// takes the chunks last to first: reload the chunk's checkpoint, recompute the
// kBwdChunk states before each token into shared memory, then walk the tokens
// backwards.  A log-gate clamped at the kernels' floor (-20) gets gradient 0
// there.
#include "common.cuh"
#include "internal.h"

namespace gdr {
namespace {

constexpr int kBwdThreads = 128;
constexpr int kBwdChunk = 16;

template <int DK>
struct BwdShape {
    static constexpr int LPR = DK / 16;          // lanes per row
    static constexpr int RB = kBwdThreads / LPR; // rows per CTA
};

struct BwdArgs {
    const void *q, *k, *v;
    const float *g, *beta, *h0;
    const int32_t *cu;
    const void *dO;
    const float *dSf;
    float *dq, *dk, *dv, *dg, *dbeta, *dh0;
    float *ckpt;
    int N, T, Hqk, H, DV;
};

// Shared memory of one CTA, in floats.
template <int DK, bool CHANNEL>
__host__ __device__ constexpr int bwd_smem_floats() {
    constexpr int CT = kBwdChunk, RB = BwdShape<DK>::RB, GD = CHANNEL ? DK : 1;
    return CT * RB * DK          // states before each token of the chunk
           + 2 * CT * DK         // k, q
           + 2 * CT * GD         // a = exp(g), and a where g is not clamped (else 0)
           + CT                  // beta
           + 2 * CT * RB         // v and dO of the CTA's rows
           + 2 * CT * DK         // dq, dk sums over the rows
           + CT * GD + CT        // dg, dbeta sums over the rows
           + (CHANNEL ? 3 : 2) * RB * DK + 2 * RB;   // one token's per-row parts
}

template <int LPR>
__device__ __forceinline__ float row_sum(float x) {
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

template <int DK, bool CHANNEL, typename IoT>
__global__ void __launch_bounds__(kBwdThreads, 1) backward_kernel(const __grid_constant__ BwdArgs A) {
    using Sh = BwdShape<DK>;
    constexpr int LPR = Sh::LPR, RB = Sh::RB, CT = kBwdChunk, GD = CHANNEL ? DK : 1;
    extern __shared__ __align__(16) float sm[];
    float *st = sm;                      // [CT][RB][DK]
    float *kc = st + CT * RB * DK;       // [CT][DK]
    float *qc = kc + CT * DK;            // [CT][DK]
    float *ac = qc + CT * DK;            // [CT][GD]
    float *am = ac + CT * GD;            // [CT][GD]
    float *bc = am + CT * GD;            // [CT]
    float *vc = bc + CT;                 // [CT][RB]
    float *oc = vc + CT * RB;            // [CT][RB]
    float *dqa = oc + CT * RB;           // [CT][DK]
    float *dka = dqa + CT * DK;          // [CT][DK]
    float *dga = dka + CT * DK;          // [CT][GD]
    float *dba = dga + CT * GD;          // [CT]
    float *pq = dba + CT;                // [RB][DK] one token's per-row parts of dq
    float *pk = pq + RB * DK;            // [RB][DK] ... of dk
    float *pg = pk + RB * DK;            // [RB][DK] ... of dg (channel gate)
    float *pb = pg + (CHANNEL ? RB * DK : 0);   // [RB] ... of dbeta
    float *ps = pb + RB;                 // [RB] ... of dg (scalar gate)

    const int nblk = (A.DV + RB - 1) / RB;
    const int nh = blockIdx.x / nblk, r0 = (blockIdx.x % nblk) * RB;
    const int n = nh / A.H, h = nh % A.H;
    const int hq = h / (A.H / A.Hqk);
    const int tid = threadIdx.x, rl = tid / LPR, p = tid % LPR;
    const int r = r0 + rl;
    const bool rv = r < A.DV;
    int a0, len;
    sequence_range(A.cu, n, A.N, A.T, a0, len);
    const int nc = (len + CT - 1) / CT;
    const IoT *q = static_cast<const IoT *>(A.q), *k = static_cast<const IoT *>(A.k);
    const IoT *v = static_cast<const IoT *>(A.v), *dO = static_cast<const IoT *>(A.dO);

    // this lane's columns: 4 (p + LPR m) + c, m, c = 0..3
    auto col = [&](int m, int c) { return 4 * (p + LPR * m) + c; };
    const size_t row_off = ((size_t)nh * A.DV + r) * DK;     // row r of (n, h) in a state array

    float s[16], ds[16];
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int c = 0; c < 4; ++c) s[4 * m + c] = (rv && A.h0 != nullptr) ? A.h0[row_off + col(m, c)] : 0.f;

    // inputs of tokens t0 .. t0 + cnt - 1 into shared memory
    auto stage = [&](int t0, int cnt, bool backward) {
        for (int i = tid; i < cnt * DK; i += kBwdThreads) {
            const int j = i / DK, c = i % DK;
            const size_t row = ((size_t)(t0 + j) * A.Hqk + hq) * DK + c;
            kc[i] = to_f32(k[row]);
            if (backward) qc[i] = to_f32(q[row]);
        }
        for (int i = tid; i < cnt * GD; i += kBwdThreads) {
            const int j = i / GD, c = i % GD;
            const float gg = A.g[((size_t)(t0 + j) * A.H + h) * GD + c];
            const float ex = __expf(clamp_log_gate(gg));
            ac[i] = ex;
            am[i] = gg > kLogGateMin ? ex : 0.f;
        }
        for (int i = tid; i < cnt; i += kBwdThreads) bc[i] = A.beta[(size_t)(t0 + i) * A.H + h];
        for (int i = tid; i < cnt * RB; i += kBwdThreads) {
            const int j = i / RB, rr = r0 + i % RB;
            const size_t at = ((size_t)(t0 + j) * A.H + h) * A.DV + rr;
            vc[i] = rr < A.DV ? to_f32(v[at]) : 0.f;
            if (backward) oc[i] = rr < A.DV ? to_f32(dO[at]) : 0.f;
        }
    };
    // one forward token on this lane's part of row r; returns x and u
    auto forward_token = [&](int j, float &x, float &u) {
        float e[16];
        x = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int cc = col(m, c);
                e[4 * m + c] = s[4 * m + c] * (CHANNEL ? ac[j * GD + cc] : ac[j]);
                x = fmaf(e[4 * m + c], kc[j * DK + cc], x);
            }
        x = row_sum<LPR>(x);
        u = bc[j] * (vc[j * RB + rl] - x);
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int c = 0; c < 4; ++c) s[4 * m + c] = fmaf(u, kc[j * DK + col(m, c)], e[4 * m + c]);
    };

    // forward sweep: checkpoint before every chunk
    for (int ch = 0; ch < nc; ++ch) {
        const int t0 = a0 + ch * CT, cnt = min(CT, a0 + len - t0);
        const size_t slot = (size_t)n + (size_t)t0 / CT;
        if (rv) {
            float *dst = A.ckpt + ((slot * A.H + h) * A.DV + r) * DK;
#pragma unroll
            for (int m = 0; m < 4; ++m)
                *reinterpret_cast<float4 *>(dst + col(m, 0)) =
                    make_float4(s[4 * m], s[4 * m + 1], s[4 * m + 2], s[4 * m + 3]);
        }
        __syncthreads();
        stage(t0, cnt, false);
        __syncthreads();
        for (int j = 0; j < cnt; ++j) {
            float x, u;
            forward_token(j, x, u);
        }
    }

    // reverse sweep
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int c = 0; c < 4; ++c) ds[4 * m + c] = (rv && A.dSf != nullptr) ? A.dSf[row_off + col(m, c)] : 0.f;
    for (int ch = nc - 1; ch >= 0; --ch) {
        const int t0 = a0 + ch * CT, cnt = min(CT, a0 + len - t0);
        const size_t slot = (size_t)n + (size_t)t0 / CT;
        if (rv) {
            const float *src = A.ckpt + ((slot * A.H + h) * A.DV + r) * DK;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 x4 = *reinterpret_cast<const float4 *>(src + col(m, 0));
                s[4 * m] = x4.x; s[4 * m + 1] = x4.y; s[4 * m + 2] = x4.z; s[4 * m + 3] = x4.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) s[i] = 0.f;
        }
        __syncthreads();
        stage(t0, cnt, true);
        __syncthreads();
        // states before each token (every thread stores and later reads only its own part)
        for (int j = 0; j < cnt; ++j) {
            float *dst = st + ((size_t)j * RB + rl) * DK;
#pragma unroll
            for (int m = 0; m < 4; ++m)
                *reinterpret_cast<float4 *>(dst + col(m, 0)) =
                    make_float4(s[4 * m], s[4 * m + 1], s[4 * m + 2], s[4 * m + 3]);
            float x, u;
            forward_token(j, x, u);
        }
        for (int j = cnt - 1; j >= 0; --j) {
            const int t = t0 + j;
            const float *sp = st + ((size_t)j * RB + rl) * DK;
#pragma unroll
            for (int i = 0; i < 16; ++i) s[i] = sp[col(i / 4, i % 4)];
            float e[16], x = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int cc = col(i / 4, i % 4);
                e[i] = s[i] * (CHANNEL ? ac[j * GD + cc] : ac[j]);
                x = fmaf(e[i], kc[j * DK + cc], x);
            }
            x = row_sum<LPR>(x);
            const float b = bc[j], vr = vc[j * RB + rl], dor = oc[j * RB + rl];
            const float u = b * (vr - x);
            float du = 0.f;
            float *myq = pq + rl * DK, *myk = pk + rl * DK, *myg = pg + rl * DK;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int cc = col(i / 4, i % 4);
                const float kk = kc[j * DK + cc];
                const float stt = fmaf(u, kk, e[i]);                 // s_t
                ds[i] = fmaf(dor, qc[j * DK + cc], ds[i]);
                myq[cc] = dor * stt;
                du = fmaf(ds[i], kk, du);
            }
            du = row_sum<LPR>(du);
            const float dx = -b * du;
            float gpart = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int cc = col(i / 4, i % 4);
                const float kk = kc[j * DK + cc];
                myk[cc] = fmaf(u, ds[i], dx * e[i]);
                const float dE = fmaf(dx, kk, ds[i]);
                const float a = CHANNEL ? ac[j * GD + cc] : ac[j];
                if constexpr (CHANNEL) myg[cc] = dE * s[i] * am[j * GD + cc];
                else gpart = fmaf(dE, s[i], gpart);
                ds[i] = dE * a;
            }
            if constexpr (!CHANNEL) gpart = row_sum<LPR>(gpart);
            if (p == 0) {
                pb[rl] = (vr - x) * du;
                if constexpr (!CHANNEL) ps[rl] = gpart * am[j];
                if (rv) A.dv[((size_t)t * A.H + h) * A.DV + r] = b * du;
            }
            __syncthreads();
            // sums over the CTA's rows, one writer per element (rows past d_v
            // hold zeros: their state, v and dO are zero)
            for (int c = tid; c < DK; c += kBwdThreads) {
                float sq = 0.f, sk = 0.f, sg = 0.f;
                for (int rr = 0; rr < RB; ++rr) {
                    sq += pq[rr * DK + c];
                    sk += pk[rr * DK + c];
                    if constexpr (CHANNEL) sg += pg[rr * DK + c];
                }
                dqa[j * DK + c] = sq;
                dka[j * DK + c] = sk;
                if constexpr (CHANNEL) dga[j * DK + c] = sg;
            }
            if (tid == kBwdThreads - 1 || (!CHANNEL && tid == kBwdThreads - 2)) {
                const float *src = tid == kBwdThreads - 1 ? pb : ps;
                float sum = 0.f;
                for (int rr = 0; rr < RB; ++rr) sum += src[rr];
                if (tid == kBwdThreads - 1) dba[j] = sum;
                else dga[j] = sum;
            }
            __syncthreads();
        }
        __syncthreads();
        for (int i = tid; i < cnt * DK; i += kBwdThreads) {
            const int j = i / DK, c = i % DK;
            const size_t at = ((size_t)(t0 + j) * A.Hqk + hq) * DK + c;
            atomicAdd(&A.dq[at], dqa[i]);
            atomicAdd(&A.dk[at], dka[i]);
        }
        for (int i = tid; i < cnt * GD; i += kBwdThreads) {
            const int j = i / GD, c = i % GD;
            atomicAdd(&A.dg[((size_t)(t0 + j) * A.H + h) * GD + c], dga[i]);
        }
        for (int i = tid; i < cnt; i += kBwdThreads)
            atomicAdd(&A.dbeta[(size_t)(t0 + i) * A.H + h], dba[i]);
    }
    if (rv && A.dh0 != nullptr) {
#pragma unroll
        for (int m = 0; m < 4; ++m)
            *reinterpret_cast<float4 *>(A.dh0 + row_off + col(m, 0)) =
                make_float4(ds[4 * m], ds[4 * m + 1], ds[4 * m + 2], ds[4 * m + 3]);
    }
}

template <int DK, bool CHANNEL, typename IoT>
cudaError_t launch_bwd_dk(const BwdArgs &A, cudaStream_t stream) {
    auto kern = backward_kernel<DK, CHANNEL, IoT>;
    const int smem = bwd_smem_floats<DK, CHANNEL>() * (int)sizeof(float);
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void *>(kern), smem);
    if (e != cudaSuccess) return e;
    const long long nblk = (A.DV + BwdShape<DK>::RB - 1) / BwdShape<DK>::RB;
    const long long blocks = (long long)A.N * A.H * nblk;
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    kern<<<(unsigned)blocks, kBwdThreads, smem, stream>>>(A);
    return cudaGetLastError();
}

template <bool CHANNEL, typename IoT>
cudaError_t launch_bwd_mode(const BwdArgs &A, int DK, cudaStream_t stream) {
    switch (DK) {
        case 16: return launch_bwd_dk<16, CHANNEL, IoT>(A, stream);
        case 32: return launch_bwd_dk<32, CHANNEL, IoT>(A, stream);
        case 64: return launch_bwd_dk<64, CHANNEL, IoT>(A, stream);
        default: return launch_bwd_dk<128, CHANNEL, IoT>(A, stream);
    }
}

}  // namespace

size_t backward_workspace_bytes(int num_seqs, int total_T, int H, int DK, int DV) {
    const size_t slots = (size_t)num_seqs + ((size_t)total_T + kBwdChunk - 1) / kBwdChunk;
    return slots * H * DV * DK * sizeof(float);
}

cudaError_t launch_backward(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const float *h0, const int32_t *cu, int num_seqs,
                            int total_T, int Hqk, int H, int DK, int DV, bool channel, bool bf16,
                            const void *dO, const float *dSf, float *dq, float *dk, float *dv,
                            float *dg, float *dbeta, float *dh0, void *workspace,
                            cudaStream_t stream) {
    const size_t T = (size_t)total_T;
    cudaError_t e = cudaSuccess;
    // the sums over rows are accumulated with atomics into zeroed outputs
    if (T > 0) {
        e = cudaMemsetAsync(dq, 0, T * Hqk * DK * sizeof(float), stream);
        if (e == cudaSuccess) e = cudaMemsetAsync(dk, 0, T * Hqk * DK * sizeof(float), stream);
        if (e == cudaSuccess)
            e = cudaMemsetAsync(dg, 0, T * H * (channel ? DK : 1) * sizeof(float), stream);
        if (e == cudaSuccess) e = cudaMemsetAsync(dbeta, 0, T * H * sizeof(float), stream);
        if (e != cudaSuccess) return e;
    }
    BwdArgs A;
    A.q = q; A.k = k; A.v = v; A.g = g; A.beta = beta; A.h0 = h0; A.cu = cu;
    A.dO = dO; A.dSf = dSf;
    A.dq = dq; A.dk = dk; A.dv = dv; A.dg = dg; A.dbeta = dbeta; A.dh0 = dh0;
    A.ckpt = static_cast<float *>(workspace);
    A.N = num_seqs; A.T = total_T; A.Hqk = Hqk; A.H = H; A.DV = DV;
    if (channel)
        return bf16 ? launch_bwd_mode<true, __nv_bfloat16>(A, DK, stream)
                    : launch_bwd_mode<true, float>(A, DK, stream);
    return bf16 ? launch_bwd_mode<false, __nv_bfloat16>(A, DK, stream)
                : launch_bwd_mode<false, float>(A, DK, stream);
}

}  // namespace gdr
