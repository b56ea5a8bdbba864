// Chunk-parallel plan of the tensor-core prefill (bf16 I/O, d_k = d_v = 128):
// two kernels instead of one, for problems with fewer (sequence, head)
// chains than the GPU has SMs.
//
// The chunk algebra is the one of the single-kernel plan (page "How the New
// Flash Models Work: Inside GLM-5.3-Flash and Qwen3.8-Flash-Next", section
// "Linear attention: a fixed-size memory in place of the cache", Gated
// DeltaNet and Kimi Delta Attention equations, rearranged per chunk of C = 64
// tokens):
//
//   T = (I + A)^-1,  W = T diag(β)(K ⊙ Γ),  Ũ = T diag(β) V      chunk-local
//   U = Ũ - W S^T,   O = (Q ⊙ Γ) S^T + (P ⊙ causal) U,
//   S' = S Diag(Γ_C) + U^T K̂                                       state chain
//
// Everything in the first line depends on one chunk only, so it runs for
// every chunk of every head at once:
//
//   prep kernel   one CTA per (chunk, sequence, head), two CTAs per SM.  It
//                 stages the bf16 tiles with TMA, forms A and P with one
//                 tcgen05 MMA, inverts I + A on CUDA cores, builds the tf32
//                 operands and forms W and Ũ with two more MMAs.  It writes a
//                 chunk record to the workspace: -W, Q̃ = Q ⊙ Γ, K̂^T and
//                 P ⊙ causal as ready-made 128-byte-swizzled shared-memory
//                 images, Ũ as plain fp32 rows, and exp(G_C).
//   chain kernel  one CTA per (sequence, head).  It keeps the fp32 state in
//                 registers (tf32 copy in TMEM) and, per chunk, bulk-copies
//                 the record into shared memory and runs only the products
//                 that need the state:
//                   S1  X^T = S (-W)^T           U^T = Ũ^T + X^T (tf32)
//                   S1' O^T = S Q̃^T              S3  ΔS = U^T K̂
//                   S2  O^T += U^T (P ⊙ causal)^T,   S = S Diag(exp(G_C)) + ΔS
//                 with the record of the next chunks already in flight.
//
// The chain kernel does per chunk what the single-kernel plan's chain group
// does; the prep work that bounds that plan's chunk period moves to
// otherwise idle SMs.  Records take 144.5 KiB per (chunk, head); problems
// whose records exceed 1 GiB run in windows of chunks, the state passing
// between windows through the workspace.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include <cstddef>

#include "common.cuh"
#include "gdr.h"
#include "internal.h"
#include "tc_ptx.cuh"
#include "chunk_common.cuh"

namespace gdr {
namespace {

using namespace tc;

constexpr uint32_t ERR_TIMEOUT_TMA = 1u, ERR_TIMEOUT_MMA = 2u, ERR_TIMEOUT_HANDOFF = 4u,
                   ERR_SMEM_ALIGN = 8u;

// ----------------------------------------------------------- chunk record ----
// Byte offsets inside one record.  The images use the layout the chain
// kernel's MMA descriptors read (128-byte rows, 16-byte chunks XOR-swizzled
// by row % 8, blocks 1024-byte aligned).
constexpr uint32_t REC_A1 = 0;          // [-W; Q̃] [tok][dk] tf32: per 32-dk block (16 KiB) the
                                        //   64 rows of -W, then the 64 rows of Q̃ (128 x 128 B)
constexpr uint32_t REC_KH = 65536;      // K̂^T [dk][tok] tf32: 2 blocks (32 tok) of 128 x 128 B
constexpr uint32_t REC_PM = 98304;      // P ⊙ causal [i][j] tf32: 2 blocks (32 j) of 64 x 128 B
constexpr uint32_t REC_UT = 114688;     // Ũ fp32: 4 blocks of 32 dv, each [tok][32] with the
                                        //   16-byte chunks of row i XOR-swizzled by i % 8
constexpr uint32_t REC_GC = 147456;     // exp(G_C): 1 float (scalar) or 128 (channel)
constexpr uint32_t REC_BYTES = 147968;
static_assert(REC_BYTES % 16 == 0 && REC_GC + 512 == REC_BYTES, "record layout");

// Byte offset of Ũ[i][dv] inside the record.
__host__ __device__ constexpr uint32_t rec_ut_offset(uint32_t i, uint32_t dv) {
    return REC_UT + (dv >> 5) * 8192 + i * 128 + (((((dv & 31) >> 2) ^ (i & 7)) << 4) | ((dv & 3) << 2));
}

// ------------------------------------------------------------ prep kernel ----
constexpr int kPrepThreads = 256;
constexpr uint32_t PO_KQ = 0;       // bf16 [K d0-63][Q d0-63][K d64-127][Q d64-127]; then V'^T tf32
constexpr uint32_t PO_V = 32768;    // bf16 [V d0-63][V d64-127]
constexpr uint32_t PO_X1 = 49152;   // scratch (A, T fp32 / channel fp16 P1 operand / slow-path G); then K'^T tf32
constexpr uint32_t PO_TM = 81920;   // inverse scratch / channel fp16 P1 operand; then T tf32
constexpr uint32_t PO_MISC = 98304;
constexpr uint32_t PREP_SMEM = PO_MISC + 2048;   // 100352: two CTAs per SM
constexpr uint32_t PT_W = 0, PT_U = 64, PREP_TMEM_COLS = 128;

struct PrepMisc {
    uint64_t bar_tma, bar_mma;
    uint32_t tmem_base;
    int abort_flag;
    int slow;                          // channel gate: A and P on CUDA cores
    int wide;                          // scalar gate: chunk decay beyond e^-80
    union alignas(16) {
        struct {
            float beta[C], G[C], gam[C], kp[C], kh[C], ieg[C];
        } s;
        struct {
            float beta[C], T0[D], T1[D];
        } c;
    } u;                               // beta comes first in both layouts
};
static_assert(sizeof(PrepMisc) <= 2048, "prep misc area overflow");
static_assert(offsetof(PrepMisc, u) % 16 == 0, "prep misc arrays misaligned");

__device__ __forceinline__ void st_global_v4(uint8_t *p, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    *reinterpret_cast<uint4 *>(p) = make_uint4(a, b, c, d);
}
__device__ __forceinline__ void st_global_b32(uint8_t *p, uint32_t a) {
    *reinterpret_cast<uint32_t *>(p) = a;
}

// Bounded wait by every thread of the block; all threads agree on stopping.
__device__ __forceinline__ bool block_wait(uint64_t *bar, uint32_t phase, int *abort_flag,
                                           uint32_t *err, uint32_t code) {
    if (!mbar_wait(bar, phase)) {
        *abort_flag = 1;
        atomicOr(err, code);
    }
    __syncthreads();
    return *reinterpret_cast<volatile int *>(abort_flag) == 0;
}

template <bool CHANNEL>
__global__ void __launch_bounds__(kPrepThreads, 2)
prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ g,
            const float *__restrict__ beta, const int32_t *__restrict__ cu, int num_seqs,
            int total_T, int Hqk, int H, int c_begin, uint8_t *__restrict__ recs,
            uint32_t *err) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = smem_u32(smem_raw);
    const int chain = blockIdx.y;
    const int h = chain % H, n = chain / H;
    const int hq = h / (H / Hqk);
    int t0, len;
    sequence_range(cu, n, num_seqs, total_T, t0, len);
    const int c = c_begin + static_cast<int>(blockIdx.x);
    if (c * C >= len) return;          // past this sequence's last chunk
    if ((sbase & 1023u) != 0) {
        if (threadIdx.x == 0) atomicOr(err, ERR_SMEM_ALIGN);
        return;
    }
    uint8_t *sm = smem_raw;
    PrepMisc *m = reinterpret_cast<PrepMisc *>(sm + PO_MISC);
    uint8_t *rec = recs + ((size_t)blockIdx.x * gridDim.y + chain) * REC_BYTES;
    const int tok0 = t0 + c * C;
    const int cl = min(C, len - c * C);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int sub = warp & 3;           // TMEM sub-partition of this warp
    const int half = warp >> 2;         // column half
    const int row = sub * 32 + lane;    // TMEM lane = matrix row
    const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;

    if (tid == 0) {
        mbar_init(&m->bar_tma, 1);
        mbar_init(&m->bar_mma, 1);
        m->abort_flag = 0;
        m->slow = 0;
        m->wide = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&m->tmem_base, PREP_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = m->tmem_base;
    if (tid == 0) {
        mbar_arrive_expect_tx(&m->bar_tma, 6 * 8192);
        tma_load_3d(sm + PO_KQ + 0, &tm_k, &m->bar_tma, 0, hq, tok0);
        tma_load_3d(sm + PO_KQ + 16384, &tm_k, &m->bar_tma, 64, hq, tok0);
        tma_load_3d(sm + PO_KQ + 8192, &tm_q, &m->bar_tma, 0, hq, tok0);
        tma_load_3d(sm + PO_KQ + 24576, &tm_q, &m->bar_tma, 64, hq, tok0);
        tma_load_3d(sm + PO_V + 0, &tm_v, &m->bar_tma, 0, h, tok0);
        tma_load_3d(sm + PO_V + 8192, &tm_v, &m->bar_tma, 64, h, tok0);
    }

    // ---- gates (overlap the tile loads); rows past the sequence end get
    //      beta = 0 and g = 0 ------------------------------------------------
    const int ch = tid & 127, hh = tid >> 7;   // channel gate: channel, token half
    float gr[32];
    if (!CHANNEL) {
        if (tid < 32) {
            const int i0 = 2 * tid, i1 = 2 * tid + 1;
            const size_t r0 = (size_t)(tok0 + i0) * H + h, r1 = (size_t)(tok0 + i1) * H + h;
            const float b0 = i0 < cl ? beta[r0] : 0.f, b1 = i1 < cl ? beta[r1] : 0.f;
            const float g0 = i0 < cl ? clamp_log_gate(g[r0]) : 0.f;
            const float g1 = i1 < cl ? clamp_log_gate(g[r1]) : 0.f;
            const float pair = g0 + g1;
            float incl = pair;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            const float G0 = incl - pair + g0, G1 = incl;
            const float Gl = __shfl_sync(0xffffffffu, incl, 31);
            m->u.s.beta[i0] = b0; m->u.s.beta[i1] = b1;
            m->u.s.G[i0] = G0; m->u.s.G[i1] = G1;
            const float e0 = __expf(G0), e1 = __expf(G1);
            m->u.s.gam[i0] = e0; m->u.s.gam[i1] = e1;
            m->u.s.kp[i0] = b0 * e0; m->u.s.kp[i1] = b1 * e1;
            m->u.s.kh[i0] = __expf(Gl - G0); m->u.s.kh[i1] = __expf(Gl - G1);
            m->u.s.ieg[i0] = __expf(-G0); m->u.s.ieg[i1] = __expf(-G1);
            if (tid == 0) {
                m->wide = (Gl < -80.f) ? 1 : 0;
                *reinterpret_cast<float *>(rec + REC_GC) = __expf(Gl);
            }
        }
    } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            const int i = hh * 32 + k;
            gr[k] = i < cl ? g[((size_t)(tok0 + i) * H + h) * D + ch] : 0.f;
        }
        gr[0] = clamp_log_gate(gr[0]);
#pragma unroll
        for (int k = 1; k < 32; ++k) gr[k] = clamp_log_gate(gr[k]) + gr[k - 1];
        if (hh == 0) m->u.c.T0[ch] = gr[31];
        else m->u.c.T1[ch] = gr[31];
        if (tid < C) m->u.c.beta[tid] = tid < cl ? beta[(size_t)(tok0 + tid) * H + h] : 0.f;
    }

    do {
        if (!block_wait(&m->bar_tma, 0, &m->abort_flag, err, ERR_TIMEOUT_TMA)) break;

        float GC = 0.f;
        if (CHANNEL) {
            // chunk-cumulative gate of this thread's tokens; reference R = G_31
            const float T0 = m->u.c.T0[ch], T1 = m->u.c.T1[ch];
            if (hh == 1) {
#pragma unroll
                for (int k = 0; k < 32; ++k) gr[k] += T0;
            }
            const float R = T0;
            GC = T0 + T1;
            if (hh == 0) *reinterpret_cast<float *>(rec + REC_GC + ch * 4) = __expf(GC);
            // fp16 P1 operands: rows [K e^{G-R}; Q e^{G-R}] (X1), K e^{R-G} (TM)
            bool bad = false;
            const uint32_t kcol = (ch >> 6) * 16384, bcol = (ch >> 6) * 8192;
            const uint32_t cch = (ch & 63) >> 3, cel = (ch & 7) * 2;
#pragma unroll 4
            for (int k = 0; k < 32; ++k) {
                const int i = hh * 32 + k;
                const uint32_t src = sbase + PO_KQ + kcol + sw128_offset(i, cch) + cel;
                const float kv = ld_shared_bf16(src), qv = ld_shared_bf16(src + 8192);
                const float up = __expf(gr[k] - R), dn = __expf(R - gr[k]);
                const float a = kv * up, b = qv * up, e = kv * dn;
                bad |= !(fabsf(a) < kF16Limit) || !(fabsf(b) < kF16Limit) ||
                       !(fabsf(e) < kF16Limit);
                st_shared_b16(sbase + PO_X1 + kcol + sw128_offset(i, cch) + cel,
                              __half_as_ushort(__float2half_rn(a)));
                st_shared_b16(sbase + PO_X1 + kcol + sw128_offset(64 + i, cch) + cel,
                              __half_as_ushort(__float2half_rn(b)));
                st_shared_b16(sbase + PO_TM + bcol + sw128_offset(i, cch) + cel,
                              __half_as_ushort(__float2half_rn(e)));
            }
            if (bad) m->slow = 1;
            fence_proxy_async();
            __syncthreads();
        }
        const bool slow = CHANNEL && m->slow != 0;

        // ---- P1: [K; Q] K^T (with the channel decays folded in) -------------
        if (!slow) {
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        if (CHANNEL) {
                            mma_f16_ss(tmem + PT_W,
                                       sw128_kmajor_desc(sbase + PO_X1 + kb * 16384 + kk * 32),
                                       sw128_kmajor_desc(sbase + PO_TM + kb * 8192 + kk * 32),
                                       IDESC_F16, (kb | kk) != 0);
                        } else {
                            const uint32_t a = sbase + PO_KQ + kb * 16384 + kk * 32;
                            mma_f16_ss(tmem + PT_W, sw128_kmajor_desc(a), sw128_kmajor_desc(a),
                                       IDESC_BF16, (kb | kk) != 0);
                        }
                    }
                mma_commit(&m->bar_mma);
            }
            if (!block_wait(&m->bar_mma, 0, &m->abort_flag, err, ERR_TIMEOUT_MMA)) break;
            tc_fence_after();
        }

        // ---- A (fp32 scratch) and P ⊙ causal (record image, tf32) -----------
        float *Af;
        float *Tf;
        float *Xs;
        if (!slow) {
            Af = reinterpret_cast<float *>(sm + PO_X1);
            Tf = reinterpret_cast<float *>(sm + PO_X1 + 16384);
            Xs = reinterpret_cast<float *>(sm + PO_TM);
            uint32_t x[32];
            tmem_ld32(tmem + lane_off + PT_W + half * 32, x);
            tmem_wait_ld();
            // exp(G_i - G_j) as a product of row and column factors while the
            // chunk's total decay stays within e^-80, else one exponential each
            const bool wide = !CHANNEL && m->wide != 0;
            const int i = row < C ? row : row - C;
            const float Gi = CHANNEL ? 0.f : m->u.s.G[i];
            const float rowf = (row < C ? m->u.s.beta[i] : 1.f) * (CHANNEL ? 1.f : m->u.s.gam[i]);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int j0 = half * 32 + q * 4;
                float cf[4] = {1.f, 1.f, 1.f, 1.f};
                if (!CHANNEL) {
                    const float4 t = *reinterpret_cast<const float4 *>(&m->u.s.ieg[j0]);
                    cf[0] = t.x; cf[1] = t.y; cf[2] = t.z; cf[3] = t.w;
                }
                float v4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = j0 + e;
                    float f = rowf * cf[e];
                    if (wide) f = (row < C ? m->u.s.beta[i] : 1.f) * __expf(Gi - m->u.s.G[j]);
                    const bool keep = row < C ? (j < i) : (j <= i);
                    v4[e] = keep ? f * __uint_as_float(x[q * 4 + e]) : 0.f;
                }
                if (row < C)
                    st4(Af, i, j0, make_float4(v4[0], v4[1], v4[2], v4[3]));
                else
                    st_global_v4(rec + REC_PM + half * 8192 + sw128_offset(i, q), to_tf32(v4[0]),
                                 to_tf32(v4[1]), to_tf32(v4[2]), to_tf32(v4[3]));
            }
        } else {
            // exact A and P on CUDA cores: G [64][128] fp32 in X1, A in TM
            float *Gs = reinterpret_cast<float *>(sm + PO_X1);
            Af = reinterpret_cast<float *>(sm + PO_TM);
            Tf = reinterpret_cast<float *>(sm + PO_X1);
            Xs = reinterpret_cast<float *>(sm + PO_X1 + 16384);
#pragma unroll
            for (int k = 0; k < 32; ++k) Gs[(hh * 32 + k) * D + ch] = gr[k];
            __syncthreads();
            for (int pr = tid; pr < C * (C + 1) / 2; pr += kPrepThreads) {
                int i = (int)((sqrtf(8.f * (float)pr + 1.f) - 1.f) * 0.5f);
                while (i * (i + 1) / 2 > pr) --i;
                while ((i + 1) * (i + 2) / 2 <= pr) ++i;
                const int j = pr - i * (i + 1) / 2;
                float dk = 0.f, dq = 0.f;
                for (int cc = 0; cc < D; ++cc) {
                    const uint32_t kc = (cc >> 6) * 16384, chk = (cc & 63) >> 3, el = (cc & 7) * 2;
                    const float ki = ld_shared_bf16(sbase + PO_KQ + kc + sw128_offset(i, chk) + el);
                    const float qi = ld_shared_bf16(sbase + PO_KQ + kc + 8192 + sw128_offset(i, chk) + el);
                    const float kj = ld_shared_bf16(sbase + PO_KQ + kc + sw128_offset(j, chk) + el);
                    const float e = __expf(Gs[i * D + cc] - Gs[j * D + cc]) * kj;
                    dk = fmaf(ki, e, dk);
                    dq = fmaf(qi, e, dq);
                }
                Af[ax(i, j)] = (j < i) ? m->u.c.beta[i] * dk : 0.f;
                st_global_b32(rec + REC_PM + (j >> 5) * 8192 + sw128_offset(i, (j & 31) >> 2) + (j & 3) * 4,
                              to_tf32(dq));
            }
            for (int e = tid; e < C * C; e += kPrepThreads) {
                const int i = e >> 6, j = e & 63;
                if (j > i) {
                    Af[ax(i, j)] = 0.f;
                    st_global_b32(rec + REC_PM + (j >> 5) * 8192 + sw128_offset(i, (j & 31) >> 2) +
                                      (j & 3) * 4,
                                  0u);
                }
            }
        }
        __syncthreads();

        // ---- T = (I + A)^-1 -> tf32 [i][j] in TM ------------------------------
        unit_lower_inverse(Af, Tf, Xs, sbase + PO_TM, tid);
        __syncthreads();

        // ---- operands, pass 1: K'^T (X1), K̂^T and Q̃ (record) from K and Q ----
        if (!CHANNEL) {
            const int i = tid & 63;
            const float kp = m->u.s.kp[i], kh = m->u.s.kh[i], gq = m->u.s.gam[i];
            const uint32_t tcol = (i >> 5) * 16384;
            const uint32_t tchunk = (i & 31) >> 2, tel = (i & 3) * 4;
#pragma unroll 1
            for (int it = 0; it < 4; ++it) {
                const int jc = (tid >> 6) + 4 * it;
                const uint32_t kb = jc >> 3, chk = jc & 7;
                float kf[8], qf[8];
                bf16x8_to_f32(ld_shared_v4(sbase + PO_KQ + kb * 16384 + sw128_offset(i, chk)), kf);
                bf16x8_to_f32(ld_shared_v4(sbase + PO_KQ + kb * 16384 + 8192 + sw128_offset(i, chk)), qf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t j = jc * 8 + e;
                    const uint32_t off = tcol + sw128_offset(j, tchunk) + tel;
                    st_shared_b32(sbase + PO_X1 + off, to_tf32(kp * kf[e]));
                    st_global_b32(rec + REC_KH + off, to_tf32(kh * kf[e]));
                }
                uint8_t *qb = rec + REC_A1 + (jc >> 2) * 16384 + 8192;
                const uint32_t qc = (jc & 3) * 2;
                st_global_v4(qb + sw128_offset(i, qc), to_tf32(gq * qf[0]), to_tf32(gq * qf[1]),
                             to_tf32(gq * qf[2]), to_tf32(gq * qf[3]));
                st_global_v4(qb + sw128_offset(i, qc + 1), to_tf32(gq * qf[4]), to_tf32(gq * qf[5]),
                             to_tf32(gq * qf[6]), to_tf32(gq * qf[7]));
            }
        } else {
            const uint32_t kcol = (ch >> 6) * 16384, cch = (ch & 63) >> 3, cel = (ch & 7) * 2;
            const uint32_t rowblk = hh * 16384;
            const uint32_t qoff = REC_A1 + (ch >> 5) * 16384 + 8192 + (ch & 3) * 4;
            const uint32_t qch = (ch & 31) >> 2;
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
                uint32_t wk[4], wh[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int k = q4 * 4 + e, i = hh * 32 + k;
                    const uint32_t src = sbase + PO_KQ + kcol + sw128_offset(i, cch) + cel;
                    const float kv = ld_shared_bf16(src), qv = ld_shared_bf16(src + 8192);
                    const float eg = __expf(gr[k]);
                    wk[e] = to_tf32(m->u.c.beta[i] * kv * eg);
                    wh[e] = to_tf32(kv * __expf(GC - gr[k]));
                    st_global_b32(rec + qoff + sw128_offset(i, qch), to_tf32(qv * eg));
                }
                st_shared_v4(sbase + PO_X1 + rowblk + sw128_offset(ch, q4), wk[0], wk[1], wk[2], wk[3]);
                st_global_v4(rec + REC_KH + rowblk + sw128_offset(ch, q4), wh[0], wh[1], wh[2], wh[3]);
            }
        }
        __syncthreads();   // K and Q are consumed: V'^T takes their place

        // ---- operands, pass 2: V'^T = (diag(β) V)^T into the K/Q area --------
        if (!CHANNEL) {
            const int i = tid & 63;
            const float bt = m->u.s.beta[i];
            const uint32_t tcol = (i >> 5) * 16384;
            const uint32_t tchunk = (i & 31) >> 2, tel = (i & 3) * 4;
#pragma unroll 1
            for (int it = 0; it < 4; ++it) {
                const int jc = (tid >> 6) + 4 * it;
                const uint32_t kb = jc >> 3, chk = jc & 7;
                float vf[8];
                bf16x8_to_f32(ld_shared_v4(sbase + PO_V + kb * 8192 + sw128_offset(i, chk)), vf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t j = jc * 8 + e;
                    st_shared_b32(sbase + PO_KQ + tcol + sw128_offset(j, tchunk) + tel,
                                  to_tf32(bt * vf[e]));
                }
            }
        } else {
            const uint32_t vcol = (ch >> 6) * 8192, cch = (ch & 63) >> 3, cel = (ch & 7) * 2;
            const uint32_t rowblk = hh * 16384;
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
                uint32_t wv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = hh * 32 + q4 * 4 + e;
                    const float vv = ld_shared_bf16(sbase + PO_V + vcol + sw128_offset(i, cch) + cel);
                    wv[e] = to_tf32(m->u.c.beta[i] * vv);
                }
                st_shared_v4(sbase + PO_KQ + rowblk + sw128_offset(ch, q4), wv[0], wv[1], wv[2], wv[3]);
            }
        }
        fence_proxy_async();
        __syncthreads();

        // ---- P2: W^T = K'^T T^T, Ũ^T = V'^T T^T --------------------------------
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t kb = k >> 2, kk = k & 3;
                const uint64_t bd = sw128_kmajor_desc(sbase + PO_TM + kb * 8192 + kk * 32);
                mma_tf32_ss(tmem + PT_W, sw128_kmajor_desc(sbase + PO_X1 + kb * 16384 + kk * 32),
                            bd, IDESC_N64, k != 0);
                mma_tf32_ss(tmem + PT_U, sw128_kmajor_desc(sbase + PO_KQ + kb * 16384 + kk * 32),
                            bd, IDESC_N64, k != 0);
            }
            mma_commit(&m->bar_mma);
        }
        if (!block_wait(&m->bar_mma, slow ? 0 : 1, &m->abort_flag, err, ERR_TIMEOUT_MMA)) break;
        tc_fence_after();

        // ---- -W (image) and Ũ (rows) into the record; thread = d row -----------
        {
            uint32_t x[32];
            tmem_ld32(tmem + lane_off + PT_W + half * 32, x);
            tmem_wait_ld();
            const uint32_t j = row;
            uint8_t *base = rec + REC_A1 + (j >> 5) * 16384 + (j & 3) * 4;
#pragma unroll
            for (int ii = 0; ii < 32; ++ii)
                st_global_b32(base + sw128_offset(half * 32 + ii, (j & 31) >> 2),
                              to_tf32(-__uint_as_float(x[ii])));
            tmem_ld32(tmem + lane_off + PT_U + half * 32, x);
            tmem_wait_ld();
#pragma unroll
            for (int ii = 0; ii < 32; ++ii)
                *reinterpret_cast<float *>(rec + rec_ut_offset(half * 32 + ii, row)) =
                    __uint_as_float(x[ii]);
        }
    } while (0);

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, PREP_TMEM_COLS);
    }
}

// ------------------------------------------- chain kernel, one head per CTA ----
// Transposed products (TMEM lane = value channel), 256 threads: thread
// (lane group, half) owns one row of S, 64 columns.
constexpr int kChainThreads = 256;
constexpr uint32_t CO_A1 = 0;         // [-W; Q̃] record images, two stages of 64 KiB
constexpr uint32_t CO_PM = 131072;    // P, two stages of 16 KiB
constexpr uint32_t CO_KH = 163840;    // K̂^T, 32 KiB
constexpr uint32_t CO_UT = 196608;    // Ũ, 32 KiB
constexpr uint32_t CO_MISC = 229376;
constexpr uint32_t CHAIN_SMEM = CO_MISC + 2048;   // 231424
// TMEM columns: O (two buffers), U, ΔS, tf32 copy of S.
constexpr uint32_t CT_O = 0, CT_U = 128, CT_DS = 256, CT_S = 384, CHAIN_TMEM_COLS = 512;

struct ChainMisc {
    uint64_t full_a1[2], full_p[2], full_u, full_k;   // record parts landed
    uint64_t bar_s1, bar_s3, bar_o;                   // MMA groups done
    uint32_t tmem_base;
    int abort_flag;
    alignas(16) float gam[2][D];                      // exp(G_C), with the P stage
};
static_assert(sizeof(ChainMisc) <= 2048, "chain misc area overflow");

// Bounded wait by all 256 threads; all agree on stopping.
__device__ __forceinline__ bool chain_wait(uint64_t *bar, uint32_t phase, ChainMisc *m,
                                           uint32_t *err, uint32_t code) {
    if (!mbar_wait(bar, phase)) {
        m->abort_flag = 1;
        atomicOr(err, code);
    }
    group_sync(1);
    return *reinterpret_cast<volatile int *>(&m->abort_flag) == 0;
}

template <bool CHANNEL>
__global__ void __launch_bounds__(kChainThreads, 1)
chain_kernel(const uint8_t *__restrict__ recs, const float *h0, float *fin, float *ws_state,
             const int32_t *__restrict__ cu, int num_seqs, int total_T, int H, int c_begin,
             int c_end, __nv_bfloat16 *__restrict__ o, uint32_t *err) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = smem_u32(smem_raw);
    const int chain = blockIdx.x, chains = gridDim.x;
    const int h = chain % H, n = chain / H;
    int t0, len;
    sequence_range(cu, n, num_seqs, total_T, t0, len);
    const int nchunks = (len + C - 1) / C;
    if (c_begin > 0 && c_begin >= nchunks) return;   // finished in an earlier window
    const int c_stop = min(c_end, nchunks);
    const int nl = max(c_stop - c_begin, 0);
    const float *s_in = c_begin == 0 ? h0 : ws_state;
    float *s_out = c_stop == nchunks ? fin : ws_state;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int sub = warp & 3;
    const int half = warp >> 2;          // state columns half*64 .. +63
    const int row = sub * 32 + lane;     // TMEM lane = value channel
    const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
    const size_t sg = (((size_t)n * H + h) * D + row) * D + half * 64;

    float S[64];
#pragma unroll
    for (int j = 0; j < 64; j += 4) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (s_in != nullptr) x = *reinterpret_cast<const float4 *>(s_in + sg + j);
        S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
    }
    if (nl == 0) {   // empty sequence: the state passes through
        if (s_out != nullptr) {
#pragma unroll
            for (int j = 0; j < 64; j += 4)
                *reinterpret_cast<float4 *>(s_out + sg + j) =
                    make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
        return;
    }
    if ((sbase & 1023u) != 0) {
        if (tid == 0) atomicOr(err, ERR_SMEM_ALIGN);
        return;
    }
    uint8_t *sm = smem_raw;
    ChainMisc *m = reinterpret_cast<ChainMisc *>(sm + CO_MISC);
    if (tid == 0) {
        mbar_init(&m->full_a1[0], 1);
        mbar_init(&m->full_a1[1], 1);
        mbar_init(&m->full_p[0], 1);
        mbar_init(&m->full_p[1], 1);
        mbar_init(&m->full_u, 1);
        mbar_init(&m->full_k, 1);
        mbar_init(&m->bar_s1, 1);
        mbar_init(&m->bar_s3, 1);
        mbar_init(&m->bar_o, 1);
        m->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&m->tmem_base, CHAIN_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = m->tmem_base;

    {   // tf32 copy of the entering state: A operand of S1 and S1'
        uint32_t r[32];
#pragma unroll
        for (int part = 0; part < 2; ++part) {
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = to_tf32(S[part * 32 + j]);
            tmem_st32(tmem + lane_off + CT_S + half * 64 + part * 32, r);
        }
        tmem_wait_st();
    }

    // Record loads, issued by thread 0 as soon as the buffer they overwrite is
    // free.  Loads per buffer are counted so that an aborted run can wait for
    // the ones still in flight before the CTA exits.
    const uint32_t gbytes = CHANNEL ? 512u : 16u;
    uint32_t issued[6] = {0, 0, 0, 0, 0, 0};
    uint64_t *bars[6] = {&m->full_a1[0], &m->full_a1[1], &m->full_p[0], &m->full_p[1], &m->full_u,
                         &m->full_k};
    auto rec_of = [&](int lc) {
        return recs + ((size_t)lc * chains + chain) * REC_BYTES;
    };
    auto load_a1 = [&](int lc) {
        const int s = lc & 1;
        mbar_arrive_expect_tx(&m->full_a1[s], 65536);
        bulk_load(sm + CO_A1 + s * 65536, rec_of(lc) + REC_A1, 65536, &m->full_a1[s]);
        ++issued[s];
    };
    auto load_p = [&](int lc) {
        const int s = lc & 1;
        const uint8_t *r = rec_of(lc);
        mbar_arrive_expect_tx(&m->full_p[s], 16384 + gbytes);
        bulk_load(sm + CO_PM + s * 16384, r + REC_PM, 16384, &m->full_p[s]);
        bulk_load(m->gam[s], r + REC_GC, gbytes, &m->full_p[s]);
        ++issued[2 + s];
    };
    auto load_u = [&](int lc) {
        mbar_arrive_expect_tx(&m->full_u, 32768);
        bulk_load(sm + CO_UT, rec_of(lc) + REC_UT, 32768, &m->full_u);
        ++issued[4];
    };
    auto load_k = [&](int lc) {
        mbar_arrive_expect_tx(&m->full_k, 32768);
        bulk_load(sm + CO_KH, rec_of(lc) + REC_KH, 32768, &m->full_k);
        ++issued[5];
    };
    auto prefetch_rec = [&](int lc) {
        if (lc < nl) {
            const uint8_t *r = rec_of(lc);
#pragma unroll
            for (int part = 0; part < 4; ++part) bulk_prefetch_l2(r + part * 36992, 36992);
        }
    };
    if (tid == 0) {
        load_a1(0);
        load_p(0);
        load_u(0);
        load_k(0);
        if (nl > 1) {
            load_a1(1);
            load_p(1);
        }
        prefetch_rec(2);
        prefetch_rec(3);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // output of a finished chunk: lane = value channel, TMEM columns = tokens
    auto store_o = [&](int cc, uint32_t col) {
        const int tok0 = t0 + cc * C;
        const int cl = min(C, len - cc * C);
        uint32_t x[32];
        tmem_ld32(tmem + lane_off + col + half * 32, x);
        tmem_wait_ld();
#pragma unroll
        for (int ii = 0; ii < 32; ++ii) {
            const int i = half * 32 + ii;
            if (i < cl)
                o[((size_t)(tok0 + i) * H + h) * D + row] = __float2bfloat16_rn(__uint_as_float(x[ii]));
        }
    };
    auto fail = [&](uint32_t code) {
        m->abort_flag = 1;
        atomicOr(err, code);
    };

    bool ok = true;
    for (int lc = 0; lc < nl; ++lc) {
        const uint32_t par = lc & 1, sph = (lc >> 1) & 1;
        const uint32_t tmO = CT_O + par * 64;
        const uint32_t a1 = sbase + CO_A1 + par * 65536;
        // The previous chunk's S1'/S2 are done: its O is readable, U (TMEM) may
        // be overwritten and its P stage takes the chunk after this one.
        if (lc >= 1) {
            if (!chain_wait(&m->bar_o, (lc - 1) & 1, m, err, ERR_TIMEOUT_MMA)) { ok = false; break; }
            tc_fence_after();
            if (tid == 0 && lc + 1 < nl) load_p(lc + 1);
        }
        if (tid == 0) {
            if (!mbar_wait(&m->full_a1[par], sph)) {
                fail(ERR_TIMEOUT_TMA);
            } else {
                tc_fence_after();
                // S1: X^T = S (-W)^T, the only product on the state's path
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    mma_tf32_ts(tmem + CT_U, tmem + CT_S + k * 8,
                                sw128_kmajor_desc(a1 + (k >> 2) * 16384 + (k & 3) * 32), IDESC_N64,
                                k != 0);
                mma_commit(&m->bar_s1);
                // S1': O^T = S Q̃^T (runs while U is formed)
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    mma_tf32_ts(tmem + tmO, tmem + CT_S + k * 8,
                                sw128_kmajor_desc(a1 + (k >> 2) * 16384 + 8192 + (k & 3) * 32),
                                IDESC_N64, k != 0);
            }
        }
        if (lc >= 1) store_o(c_begin + lc - 1, CT_O + (par ^ 1) * 64);
        if (!chain_wait(&m->bar_s1, par, m, err, ERR_TIMEOUT_MMA)) { ok = false; break; }
        tc_fence_after();
        if (!chain_wait(&m->full_u, par, m, err, ERR_TIMEOUT_TMA)) { ok = false; break; }
        {   // U = Ũ + X, rounded to tf32 in place: A operand of S3 and S2
            uint32_t x[32];
            tmem_ld32(tmem + lane_off + CT_U + half * 32, x);
            tmem_wait_ld();
#pragma unroll
            for (int jj = 0; jj < 32; ++jj)
                x[jj] = to_tf32(__uint_as_float(x[jj]) +
                                *reinterpret_cast<const float *>(
                                    sm + CO_UT + rec_ut_offset(half * 32 + jj, row) - REC_UT));
            tmem_st32(tmem + lane_off + CT_U + half * 32, x);
            tmem_wait_st();
        }
        tc_fence_before();
        group_sync(1);
        if (tid == 0) {
            if (lc + 1 < nl) load_u(lc + 1);
            tc_fence_after();
            if (!mbar_wait(&m->full_k, par) || !mbar_wait(&m->full_p[par], sph)) {
                fail(ERR_TIMEOUT_TMA);
            } else {
                // S3: ΔS = U^T K̂, then S2: O^T += U^T (P ⊙ causal)^T
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_tf32_ts(tmem + CT_DS, tmem + CT_U + k * 8,
                                sw128_kmajor_desc(sbase + CO_KH + (k >> 2) * 16384 + (k & 3) * 32),
                                IDESC_N128, k != 0);
                mma_commit(&m->bar_s3);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_tf32_ts(tmem + tmO, tmem + CT_U + k * 8,
                                sw128_kmajor_desc(sbase + CO_PM + par * 16384 + (k >> 2) * 8192 + (k & 3) * 32),
                                IDESC_N64, 1);
                mma_commit(&m->bar_o);
            }
        }
        if (!chain_wait(&m->bar_s3, par, m, err, ERR_TIMEOUT_MMA)) { ok = false; break; }
        tc_fence_after();
        if (tid == 0) {
            // S3 done: K̂ and (S1' before it) this A1 stage are consumed
            if (lc + 1 < nl) load_k(lc + 1);
            if (lc + 2 < nl) load_a1(lc + 2);
            prefetch_rec(lc + 4);
        }
        // exp(G_C) of this chunk came with its P stage
        if (!chain_wait(&m->full_p[par], sph, m, err, ERR_TIMEOUT_TMA)) { ok = false; break; }
        {   // S = S Diag(exp(G_C)) + ΔS (fp32 master), tf32 copy back to TMEM
            const float *gcb = m->gam[par];
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                uint32_t x[32];
                tmem_ld32(tmem + lane_off + CT_DS + half * 64 + part * 32, x);
                tmem_wait_ld();
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const float gc = CHANNEL ? gcb[half * 64 + part * 32 + jj] : gcb[0];
                    const float sv = fmaf(gc, S[part * 32 + jj], __uint_as_float(x[jj]));
                    S[part * 32 + jj] = sv;
                    x[jj] = to_tf32(sv);
                }
                tmem_st32(tmem + lane_off + CT_S + half * 64 + part * 32, x);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        group_sync(1);
    }
    if (ok) {
        if (chain_wait(&m->bar_o, (nl - 1) & 1, m, err, ERR_TIMEOUT_MMA)) {
            tc_fence_after();
            store_o(c_begin + nl - 1, CT_O + ((nl - 1) & 1) * 64);
        }
    }
    if (s_out != nullptr) {
#pragma unroll
        for (int j = 0; j < 64; j += 4)
            *reinterpret_cast<float4 *>(s_out + sg + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    }
    // never leave a bulk copy in flight into this CTA's shared memory: wait for
    // the last load of every buffer (a completed phase returns at once)
    if (tid == 0) {
        for (int b = 0; b < 6; ++b)
            if (issued[b] > 0) (void)mbar_wait(bars[b], (issued[b] - 1) & 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, CHAIN_TMEM_COLS);
    }
}

// ------------------------------------- chain kernel, d_v split over 4 CTAs ----
// Each CTA owns 32 value channels (a column block of S^T) of one (sequence,
// head); the products keep the 128-row M dimension on d_k or on [W; Q̃]:
//
//   M1  D1 = [-W; Q̃] S_b^T     (M = 128: rows 0-63 give X = -W S_b^T, rows 64-127
//                                give the inter-chunk output Q̃ S_b^T)
//   M2  ΔS_b^T = K̂^T U_b       (M = 128 = d_k)
//   M4  D1 += [junk; P ⊙ causal] U_b   (rows 64-127: the intra-chunk output)
//
// with U_b = Ũ_b + X (tf32) and S_b^T = S_b^T Diag(exp(G_C)) + ΔS_b^T kept in
// fp32 registers (thread = d_k row).  N = 32 for every product.  Warp roles:
// 0-3 own the state block, 4-5 form U, 6-7 store the output, 8 issues the
// MMAs, 9 loads the records; they hand off through mbarriers only (MMA
// completion frees record buffers through tcgen05.commit).
constexpr int kNB = 32;                       // value channels per CTA
constexpr int kSplitParts = D / kNB;          // CTAs per (sequence, head)
constexpr int kSplitThreads = 320;
constexpr uint32_t VO_A1 = 0;                 // [-W; Q̃], two stages of 64 KiB
constexpr uint32_t VO_KH = 131072;            // K̂^T, 32 KiB
constexpr uint32_t VO_A4 = 163840;            // per 16 KiB block: rows 0-63 a Ũ stage, rows 64-127 P
constexpr uint32_t VO_SB = 196608;            // S_b [32 dv][128 dk] tf32 image, 4 blocks of 4 KiB
constexpr uint32_t VO_UB = 212992;            // U_b^T [32 dv][64 tok] tf32 image, 2 blocks of 4 KiB
constexpr uint32_t VO_MISC = 221184;
constexpr uint32_t VSPLIT_SMEM = VO_MISC + 1024;   // 222208
constexpr uint32_t VT_D1 = 0, VT_DS = 64, VSPLIT_TMEM_COLS = 128;   // D1 buffers at 0 and 32
constexpr uint32_t IDESC_N32 = make_idesc(2, 128, 32);

struct VMisc {
    uint64_t full_a1[2], full_u[2], full_k, full_p;   // record parts landed
    uint64_t empty_a1[2], empty_u[2], empty_kp;       // record buffers free
    uint64_t bar1, bar2, bar4[2];                     // M1 / M2 / M4 done
    uint64_t u_ready, s_ready, o_free[2];             // role hand-offs
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(VMisc) <= 1024, "split misc area overflow");

// Bounded wait by a whole warp; the lanes agree on the outcome, so the
// warp-wide TMEM accesses after it stay convergent.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t phase) {
    return __all_sync(0xffffffffu, mbar_wait(bar, phase));
}

template <bool CHANNEL>
__global__ void __launch_bounds__(kSplitThreads, 1)
chain_split_kernel(const uint8_t *__restrict__ recs, const float *h0, float *fin, float *ws_state,
                   const int32_t *__restrict__ cu, int num_seqs, int total_T, int H, int c_begin,
                   int c_end, __nv_bfloat16 *__restrict__ o, uint32_t *err) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = smem_u32(smem_raw);
    const int chain = blockIdx.x / kSplitParts, part = blockIdx.x % kSplitParts;
    const int chains = gridDim.x / kSplitParts;
    const int h = chain % H, n = chain / H;
    const int dv0 = part * kNB;
    int t0, len;
    sequence_range(cu, n, num_seqs, total_T, t0, len);
    const int nchunks = (len + C - 1) / C;
    if (c_begin > 0 && c_begin >= nchunks) return;   // finished in an earlier window
    const int c_stop = min(c_end, nchunks);
    const int nl = max(c_stop - c_begin, 0);
    const float *s_in = c_begin == 0 ? h0 : ws_state;
    float *s_out = c_stop == nchunks ? fin : ws_state;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    // state entry (dv0 + j, t) of this (sequence, head) for state thread t
    const size_t sbase_g = (((size_t)n * H + h) * D + dv0) * D;

    if (nl == 0) {   // empty sequence: the state block passes through
        if (s_out != nullptr && tid < D) {
#pragma unroll 4
            for (int j = 0; j < kNB; ++j)
                s_out[sbase_g + (size_t)j * D + tid] = s_in != nullptr ? s_in[sbase_g + (size_t)j * D + tid] : 0.f;
        }
        return;
    }
    if ((sbase & 1023u) != 0) {
        if (tid == 0) atomicOr(err, ERR_SMEM_ALIGN);
        return;
    }
    uint8_t *sm = smem_raw;
    VMisc *m = reinterpret_cast<VMisc *>(sm + VO_MISC);
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&m->full_a1[s], 1);
            mbar_init(&m->full_u[s], 1);
            mbar_init(&m->empty_a1[s], 1);
            mbar_init(&m->empty_u[s], 64);
            mbar_init(&m->bar4[s], 1);
            mbar_init(&m->o_free[s], 64);
        }
        mbar_init(&m->full_k, 1);
        mbar_init(&m->full_p, 1);
        mbar_init(&m->empty_kp, 1);
        mbar_init(&m->bar1, 1);
        mbar_init(&m->bar2, 1);
        mbar_init(&m->u_ready, 64);
        mbar_init(&m->s_ready, 128);
        m->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&m->tmem_base, VSPLIT_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = m->tmem_base;
    volatile int *abort_flag = &m->abort_flag;
    auto fail = [&](uint32_t code) {
        *abort_flag = 1;
        atomicOr(err, code);
    };
    auto rec_of = [&](int lc) {
        return recs + ((size_t)lc * chains + chain) * REC_BYTES;
    };

    if (warp < 4) {
        // ====================================== state block S_b^T, row t ====
        const int t = tid;
        float S[kNB];
#pragma unroll
        for (int j = 0; j < kNB; ++j)
            S[j] = s_in != nullptr ? s_in[sbase_g + (size_t)j * D + t] : 0.f;
        const uint32_t sb = sbase + VO_SB + (t >> 5) * 4096 + (t & 3) * 4;
        const uint32_t sch = (t & 31) >> 2;
#pragma unroll
        for (int j = 0; j < kNB; ++j) st_shared_b32(sb + sw128_offset(j, sch), to_tf32(S[j]));
        fence_proxy_async();
        mbar_arrive(&m->s_ready);
        for (int lc = 0; lc < nl; ++lc) {
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            const uint8_t *r = rec_of(lc);
            const float gc = *reinterpret_cast<const float *>(r + REC_GC + (CHANNEL ? t * 4 : 0));
            if (!warp_wait(&m->bar2, lc & 1)) { fail(ERR_TIMEOUT_MMA); break; }
            tc_fence_after();
            uint32_t x[32];
            tmem_ld32(tmem + lane_off + VT_DS, x);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < kNB; ++j) {
                S[j] = fmaf(gc, S[j], __uint_as_float(x[j]));
                st_shared_b32(sb + sw128_offset(j, sch), to_tf32(S[j]));
            }
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(&m->s_ready);
        }
        if (s_out != nullptr) {
#pragma unroll
            for (int j = 0; j < kNB; ++j) s_out[sbase_g + (size_t)j * D + t] = S[j];
        }
    } else if (warp < 6) {
        // ======================================== U_b = Ũ_b + X, token i ====
        const int i = tid - 128;
        const uint32_t ub = sbase + VO_UB + (i >> 5) * 4096 + (i & 3) * 4;
        const uint32_t uch = (i & 31) >> 2;
        for (int lc = 0; lc < nl; ++lc) {
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            const uint32_t s = lc & 1;
            if (!warp_wait(&m->full_u[s], (lc >> 1) & 1)) { fail(ERR_TIMEOUT_TMA); break; }
            if (!warp_wait(&m->bar1, lc & 1)) { fail(ERR_TIMEOUT_MMA); break; }
            tc_fence_after();
            uint32_t x[32];
            tmem_ld32(tmem + lane_off + VT_D1 + s * 32, x);
            // Ũ row i of this block, 16-byte chunks swizzled by i % 8
            const uint32_t urow = sbase + VO_A4 + s * 16384 + i * 128;
            float u[kNB];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint4 v = ld_shared_v4(urow + ((q ^ (i & 7)) << 4));
                u[4 * q] = __uint_as_float(v.x); u[4 * q + 1] = __uint_as_float(v.y);
                u[4 * q + 2] = __uint_as_float(v.z); u[4 * q + 3] = __uint_as_float(v.w);
            }
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < kNB; ++j)
                st_shared_b32(ub + sw128_offset(j, uch), to_tf32(u[j] + __uint_as_float(x[j])));
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(&m->u_ready);
            mbar_arrive(&m->empty_u[s]);   // the Ũ stage is read
        }
    } else if (warp < 8) {
        // ================================ output rows (token i), 32 channels ====
        const int i = tid - 192;
        for (int lc = 0; lc < nl; ++lc) {
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            const uint32_t s = lc & 1;
            if (!warp_wait(&m->bar4[s], (lc >> 1) & 1)) { fail(ERR_TIMEOUT_MMA); break; }
            tc_fence_after();
            uint32_t x[32];
            tmem_ld32(tmem + lane_off + VT_D1 + s * 32, x);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&m->o_free[s]);
            const int cc = c_begin + lc;
            if (i < min(C, len - cc * C)) {
                uint4 *dst = reinterpret_cast<uint4 *>(o + ((size_t)(t0 + cc * C + i) * H + h) * D + dv0);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(x[8 * q + 2 * e]),
                                                                        __uint_as_float(x[8 * q + 2 * e + 1]));
                        w[e] = *reinterpret_cast<const uint32_t *>(&b2);
                    }
                    dst[q] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
    } else if (warp == 8) {
        // ======================================================= MMA issuer ====
        if (lane == 0) {
            const uint64_t d_sb = sw128_kmajor_desc(sbase + VO_SB);
            const uint64_t d_ub = sw128_kmajor_desc(sbase + VO_UB);
            const uint64_t d_kh = sw128_kmajor_desc(sbase + VO_KH);
            const uint64_t d_a4 = sw128_kmajor_desc(sbase + VO_A4);
            for (int lc = 0; lc < nl; ++lc) {
                if (*abort_flag) break;
                const uint32_t s = lc & 1, sph = (lc >> 1) & 1;
                // the buffers are normally ready long before the state block
                if (!mbar_wait_sleep(&m->full_a1[s], sph)) { fail(ERR_TIMEOUT_TMA); break; }
                if (lc >= 2 && !mbar_wait_sleep(&m->o_free[s], ((lc - 2) >> 1) & 1)) { fail(ERR_TIMEOUT_HANDOFF); break; }
                if (!mbar_wait_sleep(&m->s_ready, lc & 1)) { fail(ERR_TIMEOUT_HANDOFF); break; }
                tc_fence_after();
                const uint64_t d_a1 = sw128_kmajor_desc(sbase + VO_A1 + s * 65536);
                const uint32_t d1 = tmem + VT_D1 + s * 32;
                // descriptors advance by (bytes >> 4) in their start-address field
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    mma_tf32_ss(d1, d_a1 + (((k >> 2) * 16384 + (k & 3) * 32) >> 4),
                                d_sb + (((k >> 2) * 4096 + (k & 3) * 32) >> 4), IDESC_N32, k != 0);
                mma_commit(&m->bar1);
                mma_commit(&m->empty_a1[s]);
                if (!mbar_wait_sleep(&m->full_k, lc & 1) || !mbar_wait_sleep(&m->full_p, lc & 1)) {
                    fail(ERR_TIMEOUT_TMA);
                    break;
                }
                if (!mbar_wait_sleep(&m->u_ready, lc & 1)) { fail(ERR_TIMEOUT_HANDOFF); break; }
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_tf32_ss(tmem + VT_DS, d_kh + (((k >> 2) * 16384 + (k & 3) * 32) >> 4),
                                d_ub + (((k >> 2) * 4096 + (k & 3) * 32) >> 4), IDESC_N32, k != 0);
                mma_commit(&m->bar2);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_tf32_ss(d1, d_a4 + (((k >> 2) * 16384 + (k & 3) * 32) >> 4),
                                d_ub + (((k >> 2) * 4096 + (k & 3) * 32) >> 4), IDESC_N32, 1);
                mma_commit(&m->bar4[s]);
                mma_commit(&m->empty_kp);
            }
        }
    } else if (lane == 0) {
        // ==================================================== record loader ====
        uint32_t issued[6] = {0, 0, 0, 0, 0, 0};
        uint64_t *bars[6] = {&m->full_a1[0], &m->full_a1[1], &m->full_u[0], &m->full_u[1],
                             &m->full_k, &m->full_p};
        auto load_a1 = [&](int lc) {
            const int s = lc & 1;
            mbar_arrive_expect_tx(&m->full_a1[s], 65536);
            bulk_load(sm + VO_A1 + s * 65536, rec_of(lc) + REC_A1, 65536, &m->full_a1[s]);
            ++issued[s];
        };
        auto load_u = [&](int lc) {   // this CTA's 32-channel block of Ũ
            const int s = lc & 1;
            mbar_arrive_expect_tx(&m->full_u[s], 8192);
            bulk_load(sm + VO_A4 + s * 16384, rec_of(lc) + REC_UT + part * 8192, 8192, &m->full_u[s]);
            ++issued[2 + s];
        };
        auto load_kp = [&](int lc) {
            const uint8_t *r = rec_of(lc);
            mbar_arrive_expect_tx(&m->full_k, 32768);
            bulk_load(sm + VO_KH, r + REC_KH, 32768, &m->full_k);
            mbar_arrive_expect_tx(&m->full_p, 16384);
            bulk_load(sm + VO_A4 + 8192, r + REC_PM, 8192, &m->full_p);
            bulk_load(sm + VO_A4 + 16384 + 8192, r + REC_PM + 8192, 8192, &m->full_p);
            ++issued[4];
            ++issued[5];
        };
        auto prefetch_rec = [&](int lc) {
            if (lc < nl) {
                const uint8_t *r = rec_of(lc);
#pragma unroll
                for (int q = 0; q < 4; ++q) bulk_prefetch_l2(r + q * 36992, 36992);
            }
        };
        load_a1(0);
        load_kp(0);
        load_u(0);
        if (nl > 1) {
            load_a1(1);
            load_u(1);
        }
        prefetch_rec(1);
        prefetch_rec(2);
        // each buffer is refilled as soon as the step reading it has finished,
        // in the order those steps finish within a chunk
        for (int lc = 0; lc < nl; ++lc) {
            if (*abort_flag) break;
            const uint32_t s = lc & 1, sph = (lc >> 1) & 1;
            if (!mbar_wait_sleep(&m->empty_a1[s], sph)) { fail(ERR_TIMEOUT_MMA); break; }
            if (lc + 2 < nl) load_a1(lc + 2);
            if (!mbar_wait_sleep(&m->empty_u[s], sph)) { fail(ERR_TIMEOUT_HANDOFF); break; }
            if (lc + 2 < nl) load_u(lc + 2);
            if (!mbar_wait_sleep(&m->empty_kp, lc & 1)) { fail(ERR_TIMEOUT_MMA); break; }
            if (lc + 1 < nl) load_kp(lc + 1);
            prefetch_rec(lc + 3);
        }
        // never leave a bulk copy in flight into this CTA's shared memory
        for (int b = 0; b < 6; ++b)
            if (issued[b] > 0) (void)mbar_wait_sleep(bars[b], (issued[b] - 1) & 1);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, VSPLIT_TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host ----

constexpr size_t kHeaderBytes = 256;                        // error word
constexpr size_t kMaxRecordBytes = size_t(1) << 30;         // records per window
constexpr int kSplitMaxChains = 148;                        // one chain CTA per SM
constexpr int kSplitDvMaxChains = 148 / kSplitParts;        // d_v split: 4 CTAs a chain

struct SplitPlan {
    int chains = 0, max_chunks = 0, window = 0, windows = 0;
    size_t state_off = 0, rec_off = 0, bytes = 0;
};

bool make_split_plan(int num_seqs, int total_T, int H, SplitPlan &p) {
    const long long chains = (long long)num_seqs * H;
    if (chains < 1 || chains > kSplitMaxChains || total_T <= 0) return false;
    p.chains = (int)chains;
    p.max_chunks = (total_T + C - 1) / C;   // no sequence has more chunks
    const size_t per = (size_t)p.chains * REC_BYTES;
    const size_t fit = kMaxRecordBytes / per;
    p.window = (int)(fit < 1 ? 1 : (fit < (size_t)p.max_chunks ? fit : (size_t)p.max_chunks));
    p.windows = (p.max_chunks + p.window - 1) / p.window;
    const size_t state = p.windows > 1 ? (size_t)p.chains * D * D * sizeof(float) : 0;
    p.state_off = kHeaderBytes;
    p.rec_off = (kHeaderBytes + state + 1023) & ~size_t(1023);
    p.bytes = p.rec_off + (size_t)p.window * per;
    return true;
}

}  // namespace

size_t tcgen05_split_workspace_bytes(int num_seqs, int total_T, int H) {
    SplitPlan p;
    return make_split_plan(num_seqs, total_T, H, p) ? p.bytes : 0;
}

cudaError_t launch_prefill_split(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const float *h0, const int32_t *cu,
                                 int num_seqs, int total_T, int Hqk, int H, bool channel, void *o,
                                 float *fin, void *workspace, cudaStream_t stream) {
    SplitPlan p;
    if (!make_split_plan(num_seqs, total_T, H, p)) return cudaErrorInvalidValue;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint32_t *err = reinterpret_cast<uint32_t *>(ws);
    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(uint32_t), stream);
    if (e != cudaSuccess) return e;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, total_T, Hqk) || !make_map(&mk, k, total_T, Hqk) ||
        !make_map(&mv, v, total_T, H))
        return cudaErrorInvalidValue;
    const bool dv_split = p.chains <= kSplitDvMaxChains;
    auto prep = channel ? prep_kernel<true> : prep_kernel<false>;
    auto chain = channel ? chain_kernel<true> : chain_kernel<false>;
    auto chain_dv = channel ? chain_split_kernel<true> : chain_split_kernel<false>;
    e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PREP_SMEM);
    if (e != cudaSuccess) return e;
    if (dv_split)
        e = cudaFuncSetAttribute(chain_dv, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)VSPLIT_SMEM);
    else
        e = cudaFuncSetAttribute(chain, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)CHAIN_SMEM);
    if (e != cudaSuccess) return e;
    float *state = p.windows > 1 ? reinterpret_cast<float *>(ws + p.state_off) : nullptr;
    uint8_t *recs = ws + p.rec_off;
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(o);
    for (int w = 0; w < p.windows; ++w) {
        const int c0 = w * p.window;
        const int c1 = c0 + p.window < p.max_chunks ? c0 + p.window : p.max_chunks;
        prep<<<dim3((unsigned)(c1 - c0), (unsigned)p.chains), kPrepThreads, PREP_SMEM, stream>>>(
            mq, mk, mv, g, beta, cu, num_seqs, total_T, Hqk, H, c0, recs, err);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        if (dv_split)
            chain_dv<<<(unsigned)(p.chains * kSplitParts), kSplitThreads, VSPLIT_SMEM, stream>>>(
                recs, h0, fin, state, cu, num_seqs, total_T, H, c0, c1, out, err);
        else
            chain<<<(unsigned)p.chains, kChainThreads, CHAIN_SMEM, stream>>>(
                recs, h0, fin, state, cu, num_seqs, total_T, H, c0, c1, out, err);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace gdr
