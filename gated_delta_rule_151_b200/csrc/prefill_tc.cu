// Chunked prefill of the gated delta rule on the sm_100a tensor cores
// (tcgen05 MMA with TMEM accumulators, operands staged by TMA), bf16 I/O,
// d_k = d_v = 128, scalar gate (Gated DeltaNet).
//
// The algebra is the exact chunk rearrangement of the recurrence on the page
// "How the New Flash Models Work: Inside GLM-5.3-Flash and Qwen3.8-Flash-Next"
// (section "Linear attention: a fixed-size memory in place of the cache",
// Gated DeltaNet equation).  For a chunk of C = 64 tokens entering with state
// S (d_v x d_k), within-chunk cumulative log-gate G_i and γ_i = exp(G_i):
//
//   A  = strictly-lower( diag(β) (K K^T) ⊙ exp(G_i - G_j) ),  T = (I + A)^-1
//   W  = T diag(βγ) K,   Ũ = T diag(β) V
//   U  = Ũ - W S^T                                  (corrected values)
//   O  = diag(γ) Q S^T + (P ⊙ causal) U,  P_ij = exp(G_i - G_j) q_i . k_j
//   S' = γ_C S + U^T K̂,   K̂_j = exp(G_C - G_j) k_j
//
// Every exponent is <= 0.  The MMAs are written transposed so that the
// 128-wide d_v / d_k dimension is the M = 128 dimension (TMEM lane = row):
//
//   P1  [K;Q] K^T      bf16  M=128 N=64  K=128  -> K K^T (lanes 0-63), Q K^T (64-127)
//   P2  W^T = K'^T T^T tf32  M=128 N=64  K=64   (K' = diag(βγ) K)
//       Ũ^T = V'^T T^T tf32  M=128 N=64  K=64   (V' = diag(β) V), into the U accumulator
//   S1  U^T += S (-W)^T      A = S from TMEM, M=128 N=64 K=128
//   S1' O^T  = S Q̃^T         A = S from TMEM (Q̃ = diag(γ) Q)
//   S3  ΔS   = U^T K̂         A = U from TMEM, M=128 N=128 K=64
//   S2  O^T += U^T (P⊙causal)^T
//
// The fp32 master state lives in registers (thread = row of S, 64 columns);
// a tf32-rounded copy in TMEM is the A operand of S1/S1'.  Operands that feed
// the state update are tf32 (round-to-nearest) to keep the state within its
// error budget over thousands of chunks; Q K^T and K K^T use the exact bf16
// inputs.  CUDA cores apply the gates, build the operands in the 128-byte
// swizzled layout, and invert I + A (blocked 16 x 16 forward substitution).
//
// One CTA (8 warps) per (sequence, head).  Rows past a sequence's end get
// β = 0 and g = 0, which makes their A rows, u and gate increments vanish.
// Every mbarrier wait is bounded; on timeout the CTA records an error bit in
// the workspace word and stops.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "gdr.h"
#include "internal.h"
#include "tc_ptx.cuh"

namespace gdr {
namespace {

using namespace tc;

constexpr int C = 64;
constexpr int D = 128;
constexpr int kThreads = 256;

// Shared-memory map (byte offsets from a 1024-aligned base).
constexpr uint32_t OFF_KQ = 0;            // [K dk0-63][Q dk0-63][K dk64-127][Q dk64-127], bf16 8 KiB each
constexpr uint32_t OFF_V = 32768;         // [V dv0-63][V dv64-127]
constexpr uint32_t OFF_X1 = 49152;        // K'^T [dk][tok] tf32, then -W [tok][dk]
constexpr uint32_t OFF_X2 = 81920;        // V'^T [dv][tok] tf32
constexpr uint32_t OFF_KH = 114688;       // K̂^T [dk][tok] tf32 (A in fp32 before that)
constexpr uint32_t OFF_QT = 147456;       // Q̃ [tok][dk] tf32 (T in fp32 before that)
constexpr uint32_t OFF_PM = 180224;       // P [i][j] tf32
constexpr uint32_t OFF_TM = 196608;       // T [i][j] tf32
constexpr uint32_t OFF_MISC = 212992;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 2048 + 1024;  // + misc + alignment slack

constexpr int AF_LD = 65;                 // padded row stride of the fp32 scratch matrices

// TMEM columns.
constexpr uint32_t TM_P1 = 0, TM_W = 64, TM_U = 128, TM_O = 192, TM_DS = 256, TM_S = 384;
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t IDESC_P1 = make_idesc(1, 128, 64);    // bf16
constexpr uint32_t IDESC_N64 = make_idesc(2, 128, 64);   // tf32
constexpr uint32_t IDESC_N128 = make_idesc(2, 128, 128); // tf32

constexpr uint32_t ERR_TIMEOUT_TMA = 1u, ERR_TIMEOUT_MMA = 2u;

struct Misc {
    uint64_t bar_tma;
    uint64_t bar_mma;
    uint32_t tmem_base;
    int abort_flag;
    float G[C];      // cumulative log-gate
    float beta[C];
    float gam[C];    // exp(G_i)
    float kp[C];     // beta_i * exp(G_i)
    float kh[C];     // exp(G_C - G_i)
    float gC;        // exp(G_C)
};

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

__device__ __forceinline__ void st_shared_b32(uint32_t addr, uint32_t a) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(a) : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        f[2 * e] = __uint_as_float(w[e] << 16);
        f[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
}

// Wait on an mbarrier phase; every thread takes part so that all agree on
// whether to stop.  Returns false when the CTA must stop.
__device__ __forceinline__ bool cta_wait(uint64_t *bar, uint32_t phase, Misc *m, uint32_t *err,
                                         uint32_t code) {
    const bool ok = mbar_wait(bar, phase);
    if (!ok) {
        m->abort_flag = 1;
        atomicOr(err, code);
    }
    __syncthreads();
    return m->abort_flag == 0;
}

__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_gdn_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ g,
                      const float *__restrict__ beta, const float *h0,
                      const int32_t *__restrict__ cu, int num_seqs, int total_T, int H,
                      __nv_bfloat16 *__restrict__ o, float *fin, uint32_t *err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(sm);
    Misc *m = reinterpret_cast<Misc *>(sm + OFF_MISC);
    float *Af = reinterpret_cast<float *>(sm + OFF_KH);            // [64][65]
    float *Tf = reinterpret_cast<float *>(sm + OFF_QT);            // [64][65]
    float *Xt = reinterpret_cast<float *>(sm + OFF_QT + 64 * AF_LD * 4);  // [3][16][16]

    const int h = blockIdx.x % H;
    const int n = blockIdx.x / H;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int sub = warp & 3;          // TMEM sub-partition (lanes 32*sub .. +31)
    const int half = warp >> 2;        // which half of the columns this warp handles
    const int row = sub * 32 + lane;   // TMEM lane = matrix row
    const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;

    if (tid == 0) {
        mbar_init(&m->bar_tma, 1);
        mbar_init(&m->bar_mma, 1);
        m->abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(&m->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = m->tmem_base;

    int t0, len;
    sequence_range(cu, n, num_seqs, total_T, t0, len);

    // ---- initial state: thread owns row `row`, columns half*64 .. +63 ------
    const size_t sbase_g = (((size_t)n * H + h) * D + row) * D + half * 64;
    float S[64];
#pragma unroll
    for (int j = 0; j < 64; j += 4) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (h0 != nullptr) x = *reinterpret_cast<const float4 *>(h0 + sbase_g + j);
        S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
    }
    {
        uint32_t r[32];
#pragma unroll
        for (int part = 0; part < 2; ++part) {
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = to_tf32(S[part * 32 + j]);
            tmem_st32(tmem + lane_off + TM_S + half * 64 + part * 32, r);
        }
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();

    uint32_t ph_tma = 0, ph_mma = 0;
    bool alive = true;

    for (int c0 = 0; c0 < len && alive; c0 += C) {
        const int cl = min(C, len - c0);
        const int tok0 = t0 + c0;

        // ---- a1: stage the chunk tiles (TMA) and the masked gates ---------
        if (tid == 0) {
            fence_proxy_async();
            mbar_arrive_expect_tx(&m->bar_tma, 6 * 8192);
            tma_load_3d(sm + OFF_KQ + 0, &tm_k, &m->bar_tma, 0, h, tok0);
            tma_load_3d(sm + OFF_KQ + 16384, &tm_k, &m->bar_tma, 64, h, tok0);
            tma_load_3d(sm + OFF_KQ + 8192, &tm_q, &m->bar_tma, 0, h, tok0);
            tma_load_3d(sm + OFF_KQ + 24576, &tm_q, &m->bar_tma, 64, h, tok0);
            tma_load_3d(sm + OFF_V + 0, &tm_v, &m->bar_tma, 0, h, tok0);
            tma_load_3d(sm + OFF_V + 8192, &tm_v, &m->bar_tma, 64, h, tok0);
        }
        if (warp == 0) {
            // a2: within-chunk cumulative log-gate (lane holds tokens 2l, 2l+1)
            const int i0 = 2 * lane, i1 = 2 * lane + 1;
            const size_t r0 = (size_t)(tok0 + i0) * H + h, r1 = (size_t)(tok0 + i1) * H + h;
            const float g0 = i0 < cl ? clamp_log_gate(g[r0]) : 0.f;
            const float g1 = i1 < cl ? clamp_log_gate(g[r1]) : 0.f;
            const float b0 = i0 < cl ? beta[r0] : 0.f;
            const float b1 = i1 < cl ? beta[r1] : 0.f;
            float pair = g0 + g1;
            float incl = pair;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            const float excl = incl - pair;
            const float G0 = excl + g0, G1 = incl;
            const float GC = __shfl_sync(0xffffffffu, incl, 31);
            m->G[i0] = G0; m->G[i1] = G1;
            m->beta[i0] = b0; m->beta[i1] = b1;
            const float e0 = __expf(G0), e1 = __expf(G1);
            m->gam[i0] = e0; m->gam[i1] = e1;
            m->kp[i0] = b0 * e0; m->kp[i1] = b1 * e1;
            m->kh[i0] = __expf(GC - G0); m->kh[i1] = __expf(GC - G1);
            if (lane == 0) m->gC = __expf(GC);
        }
        alive = cta_wait(&m->bar_tma, ph_tma, m, err, ERR_TIMEOUT_TMA);
        ph_tma ^= 1;
        if (!alive) break;

        // ---- a3 (tensor part): P1 = [K;Q] K^T --------------------------------
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint32_t a = sbase + OFF_KQ + kb * 16384 + kk * 32;
                    mma_f16_ss(tmem + TM_P1, sw128_kmajor_desc(a), sw128_kmajor_desc(a), IDESC_P1,
                               (kb | kk) != 0);
                }
            mma_commit(&m->bar_mma);
        }
        alive = cta_wait(&m->bar_mma, ph_mma, m, err, ERR_TIMEOUT_MMA);
        ph_mma ^= 1;
        if (!alive) break;
        tc_fence_after();

        // ---- a3 (gates): A (fp32 scratch) and P (tf32 operand) -------------
        {
            uint32_t x[32];
            tmem_ld32(tmem + lane_off + TM_P1 + half * 32, x);
            tmem_wait_ld();
            if (row < C) {
                const int i = row;
                const float Gi = m->G[i], bi = m->beta[i];
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const int j = half * 32 + jj;
                    const float a = (j < i) ? bi * __expf(Gi - m->G[j]) * __uint_as_float(x[jj]) : 0.f;
                    Af[i * AF_LD + j] = a;
                }
            } else {
                const int i = row - C;
                const float Gi = m->G[i];
                const uint32_t rowaddr = sbase + OFF_PM + half * 8192;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int jj = q * 4 + e, j = half * 32 + jj;
                        const float p = (j <= i) ? __expf(Gi - m->G[j]) * __uint_as_float(x[jj]) : 0.f;
                        w[e] = to_tf32(p);
                    }
                    st_shared_v4(rowaddr + sw128_offset(i, q), w[0], w[1], w[2], w[3]);
                }
            }
        }
        __syncthreads();

        // ---- a4: T = (I + A)^-1 (blocked 16 x 16 forward substitution) -----
        if (tid < 64) {
            const int blk = tid >> 4, c = tid & 15, col = blk * 16 + c;
            for (int r = 0; r < 16; ++r) {
                const int ri = blk * 16 + r;
                float x;
                if (r < c) {
                    x = 0.f;
                } else if (r == c) {
                    x = 1.f;
                } else {
                    float acc = 0.f;
                    for (int s = c; s < r; ++s) acc = fmaf(Af[ri * AF_LD + blk * 16 + s], Tf[(blk * 16 + s) * AF_LD + col], acc);
                    x = -acc;
                }
                Tf[ri * AF_LD + col] = x;
            }
        }
        __syncthreads();
        for (int d = 1; d < 4; ++d) {
            const int nblk = 4 - d;
            for (int e = tid; e < nblk * 256; e += kThreads) {
                const int bi = e >> 8, r = (e >> 4) & 15, c = e & 15;
                const int I = d + bi, J = I - d;
                float acc = 0.f;
                for (int K = J; K < I; ++K)
#pragma unroll
                    for (int s = 0; s < 16; ++s)
                        acc = fmaf(Af[(I * 16 + r) * AF_LD + K * 16 + s], Tf[(K * 16 + s) * AF_LD + J * 16 + c], acc);
                Xt[bi * 256 + r * 16 + c] = acc;
            }
            __syncthreads();
            for (int e = tid; e < nblk * 256; e += kThreads) {
                const int bi = e >> 8, r = (e >> 4) & 15, c = e & 15;
                const int I = d + bi, J = I - d;
                float acc = 0.f;
                for (int s = 0; s <= r; ++s)
                    acc = fmaf(Tf[(I * 16 + r) * AF_LD + I * 16 + s], Xt[bi * 256 + s * 16 + c], acc);
                Tf[(I * 16 + r) * AF_LD + J * 16 + c] = -acc;
            }
            __syncthreads();
        }
        // T -> tf32 operand [i][j] (zero above the diagonal)
        for (int e = tid; e < C * 16; e += kThreads) {
            const int i = e >> 4, q = e & 15, j0 = q * 4;
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int j = j0 + k;
                w[k] = to_tf32(j <= i ? Tf[i * AF_LD + j] : 0.f);
            }
            st_shared_v4(sbase + OFF_TM + (j0 >> 5) * 8192 + sw128_offset(i, (j0 & 31) >> 2), w[0], w[1], w[2], w[3]);
        }
        __syncthreads();

        // ---- a5 operands: K'^T, V'^T, K̂^T (transposed) and Q̃ -------------
        {
            const int i = tid & 63;
            const float kp = m->kp[i], bt = m->beta[i], kh = m->kh[i], gq = m->gam[i];
            const uint32_t tcol = (i >> 5) * 16384;          // token block of the [d][tok] tiles
            const uint32_t tchunk = (i & 31) >> 2, tel = (i & 3) * 4;
#pragma unroll 1
            for (int it = 0; it < 4; ++it) {
                const int jc = (tid >> 6) + 4 * it;          // 8-wide d chunk 0..15
                const uint32_t kb = jc >> 3, ch = jc & 7;
                float kf[8], qf[8], vf[8];
                bf16x8_to_f32(ld_shared_v4(sbase + OFF_KQ + kb * 16384 + sw128_offset(i, ch)), kf);
                bf16x8_to_f32(ld_shared_v4(sbase + OFF_KQ + kb * 16384 + 8192 + sw128_offset(i, ch)), qf);
                bf16x8_to_f32(ld_shared_v4(sbase + OFF_V + kb * 8192 + sw128_offset(i, ch)), vf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t j = jc * 8 + e;
                    const uint32_t off = tcol + sw128_offset(j, tchunk) + tel;
                    st_shared_b32(sbase + OFF_X1 + off, to_tf32(kp * kf[e]));
                    st_shared_b32(sbase + OFF_X2 + off, to_tf32(bt * vf[e]));
                    st_shared_b32(sbase + OFF_KH + off, to_tf32(kh * kf[e]));
                }
                const uint32_t qb = sbase + OFF_QT + (jc >> 2) * 8192;
                const uint32_t qc = (jc & 3) * 2;
                st_shared_v4(qb + sw128_offset(i, qc), to_tf32(gq * qf[0]), to_tf32(gq * qf[1]),
                             to_tf32(gq * qf[2]), to_tf32(gq * qf[3]));
                st_shared_v4(qb + sw128_offset(i, qc + 1), to_tf32(gq * qf[4]), to_tf32(gq * qf[5]),
                             to_tf32(gq * qf[6]), to_tf32(gq * qf[7]));
            }
        }
        fence_proxy_async();
        __syncthreads();

        // ---- a5 (tensor part): W^T and Ũ^T ----------------------------------
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t kb = k >> 2, kk = k & 3;
                const uint64_t bd = sw128_kmajor_desc(sbase + OFF_TM + kb * 8192 + kk * 32);
                mma_tf32_ss(tmem + TM_W, sw128_kmajor_desc(sbase + OFF_X1 + kb * 16384 + kk * 32), bd,
                            IDESC_N64, k != 0);
                mma_tf32_ss(tmem + TM_U, sw128_kmajor_desc(sbase + OFF_X2 + kb * 16384 + kk * 32), bd,
                            IDESC_N64, k != 0);
            }
            mma_commit(&m->bar_mma);
        }
        alive = cta_wait(&m->bar_mma, ph_mma, m, err, ERR_TIMEOUT_MMA);
        ph_mma ^= 1;
        if (!alive) break;
        tc_fence_after();

        // -W -> [tok][dk] tf32 operand (thread = dk row of W^T)
        {
            uint32_t x[32];
            tmem_ld32(tmem + lane_off + TM_W + half * 32, x);
            tmem_wait_ld();
            const uint32_t j = row;
            const uint32_t base = sbase + OFF_X1 + (j >> 5) * 8192;
#pragma unroll
            for (int ii = 0; ii < 32; ++ii) {
                const uint32_t i = half * 32 + ii;
                st_shared_b32(base + sw128_offset(i, (j & 31) >> 2) + (j & 3) * 4,
                              to_tf32(-__uint_as_float(x[ii])));
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();

        // ---- a6/a7 (state part): U^T += S (-W)^T ; O^T = S Q̃^T ----------------
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const uint32_t off = (k >> 2) * 8192 + (k & 3) * 32;
                mma_tf32_ts(tmem + TM_U, tmem + TM_S + k * 8, sw128_kmajor_desc(sbase + OFF_X1 + off),
                            IDESC_N64, 1);
            }
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const uint32_t off = (k >> 2) * 8192 + (k & 3) * 32;
                mma_tf32_ts(tmem + TM_O, tmem + TM_S + k * 8, sw128_kmajor_desc(sbase + OFF_QT + off),
                            IDESC_N64, k != 0);
            }
            mma_commit(&m->bar_mma);
        }
        alive = cta_wait(&m->bar_mma, ph_mma, m, err, ERR_TIMEOUT_MMA);
        ph_mma ^= 1;
        if (!alive) break;
        tc_fence_after();

        // round U to tf32 in place (A operand of S2/S3)
        {
            uint32_t x[32];
            tmem_ld32(tmem + lane_off + TM_U + half * 32, x);
            tmem_wait_ld();
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) x[jj] = to_tf32(__uint_as_float(x[jj]));
            tmem_st32(tmem + lane_off + TM_U + half * 32, x);
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();

        // ---- a8 + a7: ΔS = U^T K̂ ; O^T += U^T (P⊙causal)^T -------------------
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t kb = k >> 2, kk = k & 3;
                mma_tf32_ts(tmem + TM_DS, tmem + TM_U + k * 8,
                            sw128_kmajor_desc(sbase + OFF_KH + kb * 16384 + kk * 32), IDESC_N128,
                            k != 0);
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t kb = k >> 2, kk = k & 3;
                mma_tf32_ts(tmem + TM_O, tmem + TM_U + k * 8,
                            sw128_kmajor_desc(sbase + OFF_PM + kb * 8192 + kk * 32), IDESC_N64, 1);
            }
            mma_commit(&m->bar_mma);
        }
        alive = cta_wait(&m->bar_mma, ph_mma, m, err, ERR_TIMEOUT_MMA);
        ph_mma ^= 1;
        if (!alive) break;
        tc_fence_after();

        // state update S = γ_C S + ΔS (fp32 master), tf32 copy back to TMEM
        {
            const float gC = m->gC;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                uint32_t x[32];
                tmem_ld32(tmem + lane_off + TM_DS + half * 64 + part * 32, x);
                tmem_wait_ld();
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const float s = fmaf(gC, S[part * 32 + jj], __uint_as_float(x[jj]));
                    S[part * 32 + jj] = s;
                    x[jj] = to_tf32(s);
                }
                tmem_st32(tmem + lane_off + TM_S + half * 64 + part * 32, x);
            }
            // outputs: lane = value channel, columns = tokens
            uint32_t x[32];
            tmem_ld32(tmem + lane_off + TM_O + half * 32, x);
            tmem_wait_ld();
#pragma unroll
            for (int ii = 0; ii < 32; ++ii) {
                const int i = half * 32 + ii;
                if (i < cl)
                    o[((size_t)(tok0 + i) * H + h) * D + row] = __float2bfloat16_rn(__uint_as_float(x[ii]));
            }
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();
    }

    // ---- a9: final state ----------------------------------------------------
    if (fin != nullptr) {
#pragma unroll
        for (int j = 0; j < 64; j += 4)
            *reinterpret_cast<float4 *>(fin + sbase_g + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host ----

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// [total_T, H, 128] bf16 viewed as a 3-D tensor {128, H, total_T}; box
// {64, 1, 64} with 128-byte swizzle: one 64-token x 64-channel tile.
bool make_map(CUtensorMap *map, const void *base, int total_T, int H) {
    auto enc = get_encode();
    if (enc == nullptr) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)total_T};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

bool tcgen05_prefill_available() { return true; }

bool tcgen05_prefill_serves(bool channel) { return !channel; }

size_t tcgen05_workspace_bytes(int, int, int) { return 16; }

cudaError_t launch_prefill_tcgen05(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, const float *h0, const int32_t *cu,
                                   int num_seqs, int total_T, int H, bool channel, void *o,
                                   float *fin, void *workspace, cudaStream_t stream) {
    if (channel) return cudaErrorNotSupported;
    uint32_t *err = static_cast<uint32_t *>(workspace);
    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(uint32_t), stream);
    if (e != cudaSuccess) return e;
    if ((size_t)num_seqs * H == 0) return cudaSuccess;
    if (total_T == 0) {
        // nothing to stage: the state passes through unchanged
        return launch_prefill_simt(q, k, v, g, beta, h0, cu, num_seqs, total_T, H, D, D, channel,
                                   true, o, fin, stream);
    }
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, total_T, H) || !make_map(&mk, k, total_T, H) || !make_map(&mv, v, total_T, H))
        return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(prefill_tc_gdn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const size_t blocks = (size_t)num_seqs * H;
    if (blocks > 0x7fffffffull) return cudaErrorInvalidConfiguration;
    prefill_tc_gdn_kernel<<<(unsigned)blocks, kThreads, SMEM_BYTES, stream>>>(
        mq, mk, mv, g, beta, h0, cu, num_seqs, total_T, H, static_cast<__nv_bfloat16 *>(o), fin,
        err);
    return cudaGetLastError();
}

}  // namespace gdr

// ----------------------------------------------- allocation-free variant ----
//
// Some callers cannot hand the library a workspace: they run where calling
// cudaMalloc is not allowed or not acceptable (inside a host framework that
// owns every device allocation through its own pool, in a latency-critical
// loop where an allocation would synchronise the device, or in plugin code
// with no allocator of its own).  For them the prefill's scratch -- the
// error word the tensor-core kernel's bounded waits write -- lives in the
// fixed-size device array below, which every GPU that loads this library
// holds until the process exits.

namespace gdr {
namespace {

constexpr size_t kNoAllocScratchBytes = 256;
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mutex;
void *g_noalloc_addr[kNoAllocMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device (host code only sees a stand-in symbol for the array).
cudaError_t noalloc_scratch_address(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_addr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace gdr

extern "C" gdr_status_t gdr_prefill_chunked_noalloc(
    const void *q, const void *k, const void *v, const float *g, const float *beta,
    const float *initial_state, const int32_t *cu_seqlens, int32_t num_seqs, int32_t total_T,
    int32_t H, int32_t d_k, int32_t d_v, gdr_gate_mode_t gate_mode, gdr_dtype_t io_dtype, void *o,
    float *final_state, void *stream) {
    size_t need = 0;
    gdr_status_t st = gdr_prefill_workspace_size(num_seqs, total_T, H, d_k, d_v, gate_mode,
                                                 io_dtype, &need);
    if (st != GDR_OK) return st;
    if (need > gdr::kNoAllocScratchBytes) return GDR_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (gdr::noalloc_scratch_address(&scratch) != cudaSuccess) return GDR_ERR_CUDA;
    return gdr_prefill_chunked(q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, total_T, H,
                               d_k, d_v, gate_mode, io_dtype, o, final_state, scratch,
                               gdr::kNoAllocScratchBytes, stream);
}

