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
//                 chunk record to the workspace: [-W; Q̃], K̂^T and P ⊙ causal
//                 as ready-made fp16 shared-memory operand images, each with a
//                 power-of-two scale, Ũ as fp32 rows, and exp(G_C).
//   chain kernel  one CTA per NB value channels of a (sequence, head), NB =
//                 32, 64 or 128 so that all chain CTAs fit the GPU at once.
//                 Per chunk it bulk-copies the record and runs only the
//                 products that need the state (fp16 operands, fp32
//                 accumulation, the state itself in fp32 registers), with the
//                 next records already in flight.
//
// fp16 with a per-block power-of-two scale keeps the 11-bit significand of
// tf32 at half the bytes and twice the MMA depth; the chain is bound by the
// shared-memory traffic of its operands, so halving them is what counts.
// Records take 90,640 bytes per (chunk, head); problems whose records exceed
// 1 GiB run in windows of chunks, the state passing between windows through
// the workspace.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstddef>
#include <mutex>

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
// Byte offsets inside one record.  The operand images are fp16 in the layout
// the chain kernel's MMA descriptors read: rows of 64 halves (128 bytes) whose
// 16-byte chunks are XOR-swizzled by row % 8, blocks 1024-byte aligned.  Each
// image block is scaled by a power of two 2^s chosen so that its largest
// magnitude lies in [2^14, 2^15): fp16 then carries the same 11-bit
// significand as tf32 for every value above 2^-29 of the block maximum, and
// the exponents s travel in the record.
constexpr uint32_t REC_A1 = 0;          // [-W; Q̃] [tok][dk]: 2 blocks (64 dk) of 128 rows,
                                        //   rows 0-63 -W (scale s_W), rows 64-127 Q̃ (s_Q)
constexpr uint32_t REC_KH = 32768;      // K̂^T [dk][tok]: 128 rows (s_K)
constexpr uint32_t REC_PM = 49152;      // P ⊙ causal [i][j]: 64 rows (s_P)
constexpr uint32_t REC_UT = 57344;      // Ũ fp32: 4 blocks of 32 dv, each [tok][32] with the
                                        //   16-byte chunks of row i XOR-swizzled by i % 8
constexpr uint32_t REC_GC = 90112;      // exp(G_C): 1 float (scalar) or 128 (channel)
constexpr uint32_t REC_EX = 90624;      // int32 {s_W, s_Q, s_K, s_P}
constexpr uint32_t REC_BYTES = 90640;
static_assert(REC_BYTES % 16 == 0 && REC_EX + 16 == REC_BYTES, "record layout");

// Byte offset of fp16 element (r, c) (c < 64) inside a block of 128-byte rows.
__host__ __device__ constexpr uint32_t h16_offset(uint32_t r, uint32_t c) {
    return r * 128u + ((((c >> 3) ^ (r & 7u)) & 7u) << 4) + (c & 7u) * 2u;
}

// Byte offset of Ũ[i][dv] inside the record.
__host__ __device__ constexpr uint32_t rec_ut_offset(uint32_t i, uint32_t dv) {
    return REC_UT + (dv >> 5) * 8192 + i * 128 + (((((dv & 31) >> 2) ^ (i & 7)) << 4) | ((dv & 3) << 2));
}

// Scale exponent s for a block whose largest magnitude is mx: mx 2^s lies in
// [2^14, 2^15).  Zero, subnormal-only or non-finite maxima give safe values;
// s is clamped to [-100, 100] so that 2^s and 2^-s stay normal floats.
__device__ __forceinline__ int scale_exp(float mx) {
    if (!(mx > 0.f) || !(mx < 3.0e38f)) return 0;
    const int e = (int)((__float_as_uint(mx) >> 23) & 255u) - 127;
    return min(max(14 - e, -100), 100);
}

// 2^s for |s| <= 126.
__device__ __forceinline__ float exp2i(int s) { return __int_as_float((127 + s) << 23); }

__device__ __forceinline__ uint16_t f2h_bits(float x) { return __half_as_ushort(__float2half_rn(x)); }

__device__ __forceinline__ uint32_t f2h2_bits(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
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
    float red[2][8];                   // per-warp maxima for the image scales
};
static_assert(sizeof(PrepMisc) <= 2048, "prep misc area overflow");
static_assert(offsetof(PrepMisc, u) % 16 == 0, "prep misc arrays misaligned");

__device__ __forceinline__ void st_global_v4(uint8_t *p, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    *reinterpret_cast<uint4 *>(p) = make_uint4(a, b, c, d);
}
__device__ __forceinline__ void st_global_b16(uint8_t *p, uint16_t a) {
    *reinterpret_cast<uint16_t *>(p) = a;
}

// Scale exponents of two blocks from every thread's largest |value| of each
// (a, b >= 0); all 256 threads call it (two __syncthreads inside).
__device__ __forceinline__ void block_scale2(float a, float b, float (*red)[8], int &sa, int &sb) {
    const uint32_t ua = __reduce_max_sync(0xffffffffu, __float_as_uint(a));
    const uint32_t ub = __reduce_max_sync(0xffffffffu, __float_as_uint(b));
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
        red[0][w] = __uint_as_float(ua);
        red[1][w] = __uint_as_float(ub);
    }
    __syncthreads();
    float ma = 0.f, mb = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        ma = fmaxf(ma, red[0][k]);
        mb = fmaxf(mb, red[1][k]);
    }
    __syncthreads();
    sa = scale_exp(ma);
    sb = scale_exp(mb);
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
        float kmax = 0.f, qmax = 0.f;   // channel gate: this thread's largest |k| and |q|
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
                kmax = fmaxf(kmax, fabsf(kv));
                qmax = fmaxf(qmax, fabsf(qv));
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

        // ---- A (fp32 scratch) and P ⊙ causal (record image, fp16) -----------
        int sP = 0, sQ = 0, sK = 0, sW = 0;   // record image scale exponents
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
            float pv[32];   // P row i, columns half*32 .. +31 (rows 64-127 of P1)
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
                if (row < C) {
                    st4(Af, i, j0, make_float4(v4[0], v4[1], v4[2], v4[3]));
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e) pv[q * 4 + e] = v4[e];
                }
            }
            float pm = 0.f;
            if (row >= C) {
#pragma unroll
                for (int e = 0; e < 32; ++e) pm = fmaxf(pm, fabsf(pv[e]));
            }
            int unused;
            block_scale2(pm, 0.f, m->red, sP, unused);
            if (row >= C) {
                const float f = exp2i(sP);
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const float *v = pv + c4 * 8;
                    st_global_v4(rec + REC_PM + i * 128 + ((((half * 4 + c4) ^ (i & 7)) & 7) << 4),
                                 f2h2_bits(v[0] * f, v[1] * f), f2h2_bits(v[2] * f, v[3] * f),
                                 f2h2_bits(v[4] * f, v[5] * f), f2h2_bits(v[6] * f, v[7] * f));
                }
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
            // pair pr = i (i + 1) / 2 + j (j <= i); each thread keeps its P values
            // until the block's scale is known
            constexpr int kPairIters = (C * (C + 1) / 2 + kPrepThreads - 1) / kPrepThreads;
            auto pair_ij = [](int pr, int &i, int &j) {
                i = (int)((sqrtf(8.f * (float)pr + 1.f) - 1.f) * 0.5f);
                while (i * (i + 1) / 2 > pr) --i;
                while ((i + 1) * (i + 2) / 2 <= pr) ++i;
                j = pr - i * (i + 1) / 2;
            };
            float dqs[kPairIters];
            float pm = 0.f;
#pragma unroll
            for (int it = 0; it < kPairIters; ++it) {
                const int pr = tid + it * kPrepThreads;
                dqs[it] = 0.f;
                if (pr < C * (C + 1) / 2) {
                    int i, j;
                    pair_ij(pr, i, j);
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
                    dqs[it] = dq;
                    pm = fmaxf(pm, fabsf(dq));
                }
            }
            for (int e = tid; e < C * C; e += kPrepThreads) {
                const int i = e >> 6, j = e & 63;
                if (j > i) {
                    Af[ax(i, j)] = 0.f;
                    st_global_b16(rec + REC_PM + h16_offset(i, j), 0);
                }
            }
            int unused;
            block_scale2(pm, 0.f, m->red, sP, unused);
            const float f = exp2i(sP);
#pragma unroll
            for (int it = 0; it < kPairIters; ++it) {
                const int pr = tid + it * kPrepThreads;
                if (pr < C * (C + 1) / 2) {
                    int i, j;
                    pair_ij(pr, i, j);
                    st_global_b16(rec + REC_PM + h16_offset(i, j), f2h_bits(dqs[it] * f));
                }
            }
        }
        __syncthreads();

        // ---- T = (I + A)^-1 -> tf32 [i][j] in TM ------------------------------
        unit_lower_inverse(Af, Tf, Xs, sbase + PO_TM, tid);
        __syncthreads();

        // ---- operands, pass 1: K'^T (X1, tf32), K̂^T and Q̃ (record, fp16) ------
        if (!CHANNEL) {
            const int i = tid & 63;
            const float kp = m->u.s.kp[i], kh = m->u.s.kh[i], gq = m->u.s.gam[i];
            // the chunk's largest |K̂| and |Q̃| set their image scales
            float mk = 0.f, mq = 0.f;
#pragma unroll 1
            for (int it = 0; it < 4; ++it) {
                const int jc = (tid >> 6) + 4 * it;
                const uint32_t kb = jc >> 3, chk = jc & 7;
                float kf[8], qf[8];
                bf16x8_to_f32(ld_shared_v4(sbase + PO_KQ + kb * 16384 + sw128_offset(i, chk)), kf);
                bf16x8_to_f32(ld_shared_v4(sbase + PO_KQ + kb * 16384 + 8192 + sw128_offset(i, chk)), qf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    mk = fmaxf(mk, fabsf(kh * kf[e]));
                    mq = fmaxf(mq, fabsf(gq * qf[e]));
                }
            }
            block_scale2(mk, mq, m->red, sK, sQ);
            const float fk = exp2i(sK), fq = exp2i(sQ);
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
                    st_shared_b32(sbase + PO_X1 + tcol + sw128_offset(j, tchunk) + tel, to_tf32(kp * kf[e]));
                    st_global_b16(rec + REC_KH + h16_offset(j, i), f2h_bits(kh * kf[e] * fk));
                }
                // Q̃ row 64 + i, channels jc*8 .. +7: one 16-byte chunk
                st_global_v4(rec + REC_A1 + kb * 16384 + (64 + i) * 128 + (((chk ^ (i & 7)) & 7) << 4),
                             f2h2_bits(gq * qf[0] * fq, gq * qf[1] * fq),
                             f2h2_bits(gq * qf[2] * fq, gq * qf[3] * fq),
                             f2h2_bits(gq * qf[4] * fq, gq * qf[5] * fq),
                             f2h2_bits(gq * qf[6] * fq, gq * qf[7] * fq));
            }
        } else {
            const uint32_t kcol = (ch >> 6) * 16384, cch = (ch & 63) >> 3, cel = (ch & 7) * 2;
            // scales from bounds: |K̂| <= max|k| e^{max(G_C - G)}, |Q̃| <= max|q| e^{max G};
            // a bound above the true maximum only moves values down within fp16's
            // normal range, so the precision is the same
            float dk = -3.0e38f, dq = -3.0e38f;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                dk = fmaxf(dk, GC - gr[k]);
                dq = fmaxf(dq, gr[k]);
            }
            block_scale2(kmax * __expf(dk), qmax * __expf(dq), m->red, sK, sQ);
            const float fk = exp2i(sK), fq = exp2i(sQ);
            const uint32_t rowblk = hh * 16384;
            uint8_t *qdst = rec + REC_A1 + (ch >> 6) * 16384;
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {   // tokens hh*32 + c8*8 .. +7
                float wh[8];
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    const int q4 = c8 * 2 + q2;
                    uint32_t wk[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int k = q4 * 4 + e, i = hh * 32 + k;
                        const uint32_t src = sbase + PO_KQ + kcol + sw128_offset(i, cch) + cel;
                        const float kv = ld_shared_bf16(src), qv = ld_shared_bf16(src + 8192);
                        const float eg = __expf(gr[k]);
                        wk[e] = to_tf32(m->u.c.beta[i] * kv * eg);
                        wh[q2 * 4 + e] = kv * __expf(GC - gr[k]) * fk;
                        st_global_b16(qdst + h16_offset(64 + i, ch & 63), f2h_bits(qv * eg * fq));
                    }
                    st_shared_v4(sbase + PO_X1 + rowblk + sw128_offset(ch, q4), wk[0], wk[1], wk[2], wk[3]);
                }
                // K̂^T row ch, tokens hh*32 + c8*8 .. +7: one 16-byte chunk
                st_global_v4(rec + REC_KH + ch * 128 + ((((hh * 4 + c8) ^ (ch & 7)) & 7) << 4),
                             f2h2_bits(wh[0], wh[1]), f2h2_bits(wh[2], wh[3]), f2h2_bits(wh[4], wh[5]),
                             f2h2_bits(wh[6], wh[7]));
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

        // ---- -W (fp16 image) and Ũ (fp32 rows) into the record; thread = d row --
        {
            uint32_t x[32];
            tmem_ld32(tmem + lane_off + PT_W + half * 32, x);
            tmem_wait_ld();
            float mw = 0.f;
#pragma unroll
            for (int ii = 0; ii < 32; ++ii) mw = fmaxf(mw, fabsf(__uint_as_float(x[ii])));
            int unused;
            block_scale2(mw, 0.f, m->red, sW, unused);
            const float fw = -exp2i(sW);
            const uint32_t j = row;
            uint8_t *base = rec + REC_A1 + (j >> 6) * 16384;
#pragma unroll
            for (int ii = 0; ii < 32; ++ii)
                st_global_b16(base + h16_offset(half * 32 + ii, j & 63), f2h_bits(__uint_as_float(x[ii]) * fw));
            if (tid == 0)
                *reinterpret_cast<int4 *>(rec + REC_EX) = make_int4(sW, sQ, sK, sP);
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

// ----------------------------------------------------------- chain kernel ----
// Each CTA owns NB value channels (a column block of S^T) of one (sequence,
// head); the (D / NB) CTAs of a head run in lockstep on the same records.
// Every product keeps the 128-row M dimension on [W; Q̃] or on d_k, with
// fp16 operands (K = 16 per MMA) and fp32 accumulators:
//
//   M1  D1 = [-W; Q̃] S_b^T          rows 0-63: X = -W S_b^T
//                                   rows 64-127: the inter-chunk output Q̃ S_b^T
//   M2  D2 = K̂^T U_b                ΔS_b^T
//   M4  D4 = [junk; P ⊙ causal] U_b rows 64-127: the intra-chunk output
//
// U_b = Ũ_b + X and S_b^T = S_b^T Diag(exp(G_C)) + ΔS_b^T are formed in fp32
// (the state block stays in registers, thread = d_k row) and written back as
// fp16 images with a fresh power-of-two scale each chunk; every accumulator
// is unscaled by the exponents of its two operands.  Warp roles: state
// block, U (tokens 0-63 of D1), output (tokens 64-127 of D1 and D4), the MMA
// issuer and the record loader, handing off through mbarriers only; record
// buffers are freed by tcgen05.commit of the MMAs that read them.
template <int NB>
struct Chain {
    static constexpr int kSW = NB <= 64 ? 4 : 8;         // state warps
    static constexpr int kCS = NB * 4 / kSW;              // state columns per thread
    static constexpr int kSets = NB <= 64 ? 1 : 2;        // sets of (2 U warps, 2 output warps)
    static constexpr int kCU = NB / kSets;                // U / output columns per thread
    static constexpr int kIssuer = kSW + 4 * kSets;       // MMA issuer warp; the loader follows
    static constexpr int kThreads = 32 * (kIssuer + 2);
    static constexpr bool kDB = NB <= 64;                 // two K̂/P stages and O buffers
    static constexpr int kStages = kDB ? 2 : 1;
    static constexpr uint32_t A1 = 0;                     // [-W; Q̃], 2 stages of 32 KiB
    static constexpr uint32_t KH = 65536;                 // K̂^T, 16 KiB per stage
    static constexpr uint32_t A4 = KH + kStages * 16384;  // [junk; P], 16 KiB per stage
    static constexpr uint32_t UT = A4 + kStages * 16384;  // Ũ fp32, 2 stages of 256 NB bytes
    static constexpr uint32_t SB = UT + 512 * NB;         // S_b image [NB][128], 256 NB bytes
    static constexpr uint32_t UB = SB + 256 * NB;         // U_b^T image [NB][64], 128 NB bytes
    static constexpr uint32_t MISC = UB + 128 * NB;
    static constexpr uint32_t SMEM = MISC + 1024;
    static constexpr uint32_t TD1 = 0;                    // per O buffer
    static constexpr uint32_t TD4 = kStages * NB;         // per O buffer
    static constexpr uint32_t TD2 = 2 * kStages * NB;
    static constexpr uint32_t TCOLS = TD2 + NB <= 256 ? 256 : 512;
    // fp16 x fp16 -> fp32, B (the S and U images) MN-major
    static constexpr uint32_t IDESC = make_idesc(0, 128, NB) | (1u << 16);
    static_assert(SMEM <= 232448 && TD2 + NB <= 512, "chain kernel does not fit");
    // the S and U images are MN-major with one 64-byte row (32 channels) per K index
    static_assert(NB == 32, "MN-major images hold 32 value channels");
};

struct ChainMisc {
    uint64_t full_a1[2], full_u[2], full_kp[2];     // record parts landed
    uint64_t empty_a1[2], empty_u[2], empty_kp[2];  // record buffers free
    uint64_t bar1, bar2, bar4[2];                   // M1 / M2 / M4 done
    uint64_t s_ready, u_ready, o_free[2], osc_full[2];
    uint32_t tmem_base;
    int abort_flag;
    int es[4];                  // S image exponent, per chunk mod 4
    int dsx[2][2];              // {s_K, s_U}, per chunk parity
    int osx[2][4];              // {s_Q, s_S, s_P, s_U}, per chunk parity
    alignas(16) int ex[2][4];   // record exponents {s_W, s_Q, s_K, s_P}, with the Ũ stage
    float red_s[2][8], red_u[2][4];
};
static_assert(sizeof(ChainMisc) <= 1024, "chain misc area overflow");

// Bounded wait by a whole warp; the lanes agree on the outcome, so the
// warp-wide TMEM accesses after it stay convergent.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t phase) {
    return __all_sync(0xffffffffu, mbar_wait_sleep(bar, phase));
}

// Named barrier over `nthreads` threads that also ORs a flag across them.
__device__ __forceinline__ bool named_sync_or(int id, int nthreads, bool flag) {
    uint32_t any;
    asm volatile(
        "{\n\t.reg .pred pc, pr;\n\t"
        "setp.ne.u32 pc, %1, 0;\n\t"
        "barrier.red.or.pred pr, %2, %3, pc;\n\t"
        "selp.u32 %0, 1, 0, pr;\n\t}"
        : "=r"(any)
        : "r"((uint32_t)flag), "r"(id), "r"(nthreads)
        : "memory");
    return any != 0;
}

// Largest |value| over a role's warps -> the role-wide scale exponent.  The
// barrier also agrees on stopping: every warp of the role calls this once
// per chunk, even after a failed wait, and all of them see `stop` true if
// any thread passed stop = true or the CTA's abort flag was set before.
__device__ __forceinline__ int role_scale(float mx, float *slots, int slot, int nwarps, int bar_id,
                                          bool &stop, volatile int *abort_flag) {
    const uint32_t wm = __reduce_max_sync(0xffffffffu, __float_as_uint(mx));
    if ((threadIdx.x & 31) == 0) slots[slot] = __uint_as_float(wm);
    stop = named_sync_or(bar_id, nwarps * 32, stop || *abort_flag != 0);
    float bm = 0.f;
    for (int w = 0; w < nwarps; ++w) bm = fmaxf(bm, slots[w]);
    return scale_exp(bm);
}

template <bool CHANNEL, int NB>
__global__ void __launch_bounds__(Chain<NB>::kThreads, 1)
chain_kernel(const uint8_t *__restrict__ recs, const float *h0, float *fin, float *ws_state,
             const int32_t *__restrict__ cu, int num_seqs, int total_T, int H, int c_begin,
             int c_end, __nv_bfloat16 *__restrict__ o, uint32_t *err) {
    using K = Chain<NB>;
    constexpr int kParts = D / NB;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = smem_u32(smem_raw);
    const int chain = blockIdx.x / kParts, part = blockIdx.x % kParts;
    const int chains = gridDim.x / kParts;
    const int h = chain % H, n = chain / H;
    const int dv0 = part * NB;
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
    // entry (dv0 + j, t) of this (sequence, head)'s state
    const size_t sg = (((size_t)n * H + h) * D + dv0) * D;

    if (nl == 0) {   // empty sequence: the state block passes through
        if (s_out != nullptr && tid < D) {
            for (int j = 0; j < NB; ++j)
                s_out[sg + (size_t)j * D + tid] = s_in != nullptr ? s_in[sg + (size_t)j * D + tid] : 0.f;
        }
        return;
    }
    if ((sbase & 1023u) != 0) {
        if (tid == 0) atomicOr(err, ERR_SMEM_ALIGN);
        return;
    }
    uint8_t *sm = smem_raw;
    ChainMisc *m = reinterpret_cast<ChainMisc *>(sm + K::MISC);
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&m->full_a1[s], 1);
            mbar_init(&m->full_u[s], 1);
            mbar_init(&m->full_kp[s], 1);
            mbar_init(&m->empty_a1[s], 1);
            mbar_init(&m->empty_u[s], 64 * K::kSets);
            mbar_init(&m->empty_kp[s], 1);
            mbar_init(&m->bar4[s], 1);
            mbar_init(&m->o_free[s], 64 * K::kSets);
            mbar_init(&m->osc_full[s], 64 * K::kSets);
        }
        mbar_init(&m->bar1, 1);
        mbar_init(&m->bar2, 1);
        mbar_init(&m->s_ready, 32 * K::kSW);
        mbar_init(&m->u_ready, 64 * K::kSets);
        m->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&m->tmem_base, K::TCOLS);
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

    if (warp < K::kSW) {
        // ================================== state block S_b^T, thread = d_k row ====
        const int sub = warp & 3, cg = warp >> 2;
        const int t = sub * 32 + lane;
        const int c0 = cg * K::kCS;
        const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
        float S[K::kCS];
#pragma unroll
        for (int j = 0; j < K::kCS; ++j)
            S[j] = s_in != nullptr ? s_in[sg + (size_t)(c0 + j) * D + t] : 0.f;
        // fp16 image of the state block for chunk lc (MN-major: row t holds the 32
        // channels of d_k index t), with its scale exponent
        const uint32_t srow = sbase + K::SB + t * 64;
        bool stop = false;
        auto publish = [&](int lc) {
            float mx = 0.f;
#pragma unroll
            for (int j = 0; j < K::kCS; ++j) mx = fmaxf(mx, fabsf(S[j]));
            const int sS = role_scale(mx, m->red_s[lc & 1], warp, K::kSW, 1, stop, abort_flag);
            const float f = exp2i(sS);
#pragma unroll
            for (int c = 0; c < 4; ++c)
                st_shared_v4(srow + ((c ^ ((t >> 1) & 3)) << 4), f2h2_bits(S[8 * c] * f, S[8 * c + 1] * f),
                             f2h2_bits(S[8 * c + 2] * f, S[8 * c + 3] * f), f2h2_bits(S[8 * c + 4] * f, S[8 * c + 5] * f),
                             f2h2_bits(S[8 * c + 6] * f, S[8 * c + 7] * f));
            if (tid == 0) m->es[lc & 3] = sS;
            fence_proxy_async();
            mbar_arrive(&m->s_ready);
        };
        publish(0);
        for (int lc = 0; lc < nl && !stop; ++lc) {
            const float gc =
                *reinterpret_cast<const float *>(rec_of(lc) + REC_GC + (CHANNEL ? t * 4 : 0));
            // u_ready publishes the ΔS exponents; M2 done gives ΔS.  A failed wait
            // still takes part in the role's barrier below.
            if (!warp_wait(&m->u_ready, lc & 1)) { fail(ERR_TIMEOUT_HANDOFF); stop = true; }
            if (!stop && !warp_wait(&m->bar2, lc & 1)) { fail(ERR_TIMEOUT_MMA); stop = true; }
            if (!stop) {
                tc_fence_after();
                const float f1 = exp2i(-m->dsx[lc & 1][0]), f2 = exp2i(-m->dsx[lc & 1][1]);
#pragma unroll
                for (int p = 0; p < K::kCS / 16; ++p) {
                    uint32_t x[16];
                    tmem_ld16(tmem + lane_off + K::TD2 + c0 + p * 16, x);
                    tmem_wait_ld();
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj)
                        S[p * 16 + jj] = fmaf(gc, S[p * 16 + jj], __uint_as_float(x[jj]) * f1 * f2);
                }
                tc_fence_before();
            }
            if (lc + 1 < nl) publish(lc + 1);
        }
        if (s_out != nullptr) {
#pragma unroll
            for (int j = 0; j < K::kCS; ++j) s_out[sg + (size_t)(c0 + j) * D + t] = S[j];
        }
    } else if (warp < K::kIssuer) {
        const int set = (warp - K::kSW) >> 2, r = (warp - K::kSW) & 3;
        const int c0 = set * K::kCU;
        const uint32_t lane_off = static_cast<uint32_t>(r * 32) << 16;
        if (r < 2) {
            // ===================================== U_b = Ũ_b + X, thread = token i ====
            const int i = r * 32 + lane;
            const uint32_t urow_img = sbase + K::UB + i * 64;   // MN-major: row i = token
            bool stop = false;
            for (int lc = 0; lc < nl && !stop; ++lc) {
                const uint32_t s = lc & 1;
                const uint32_t b = K::kDB ? (lc & 1) : 0;
                // a failed wait still takes part in the role's barrier below
                if (!warp_wait(&m->full_u[s], (lc >> 1) & 1)) { fail(ERR_TIMEOUT_TMA); stop = true; }
                if (!stop && !warp_wait(&m->s_ready, lc & 1)) { fail(ERR_TIMEOUT_HANDOFF); stop = true; }
                if (!stop && !warp_wait(&m->bar1, lc & 1)) { fail(ERR_TIMEOUT_MMA); stop = true; }
                if (!stop) tc_fence_after();
                const int sW = m->ex[s][0], sQ = m->ex[s][1], sK = m->ex[s][2], sP = m->ex[s][3];
                const int sS = m->es[lc & 3];
                const float fa = exp2i(-sW), fb = exp2i(-sS);
                // U = Ũ + X in fp32 (this thread's token row, 32 channels)
                float u[32];
                float mx = 0.f;
                if (!stop) {
                    uint32_t x[32];
                    tmem_ld32(tmem + lane_off + K::TD1 + b * NB, x);
                    const uint32_t urow = sbase + K::UT + s * (256 * NB) + i * 128;
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const uint4 v = ld_shared_v4(urow + ((q ^ (i & 7)) << 4));
                        const float w[4] = {__uint_as_float(v.x), __uint_as_float(v.y),
                                            __uint_as_float(v.z), __uint_as_float(v.w)};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            u[q * 4 + e] = w[e] + __uint_as_float(x[q * 4 + e]) * fa * fb;
                            mx = fmaxf(mx, fabsf(u[q * 4 + e]));
                        }
                    }
                }
                const int sU = role_scale(mx, m->red_u[lc & 1], set * 2 + r, 2 * K::kSets, 2, stop,
                                          abort_flag);
                if (stop) break;
                const float fu = exp2i(sU);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    st_shared_v4(urow_img + ((c ^ ((i >> 1) & 3)) << 4), f2h2_bits(u[8 * c] * fu, u[8 * c + 1] * fu),
                                 f2h2_bits(u[8 * c + 2] * fu, u[8 * c + 3] * fu),
                                 f2h2_bits(u[8 * c + 4] * fu, u[8 * c + 5] * fu),
                                 f2h2_bits(u[8 * c + 6] * fu, u[8 * c + 7] * fu));
                if (i == 0 && set == 0) {
                    m->dsx[lc & 1][0] = sK;
                    m->dsx[lc & 1][1] = sU;
                    m->osx[lc & 1][0] = sQ;
                    m->osx[lc & 1][1] = sS;
                    m->osx[lc & 1][2] = sP;
                    m->osx[lc & 1][3] = sU;
                }
                fence_proxy_async();
                tc_fence_before();
                mbar_arrive(&m->u_ready);
                mbar_arrive(&m->empty_u[s]);   // this Ũ stage (and its exponents) is read
                mbar_arrive(&m->osc_full[lc & 1]);
            }
        } else {
            // ====================== output rows (token i = TMEM lane - 64), NB/kSets channels ====
            const int i = (r - 2) * 32 + lane;
            for (int lc = 0; lc < nl; ++lc) {
                if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
                const uint32_t b = K::kDB ? (lc & 1) : 0;
                const uint32_t bph = K::kDB ? ((lc >> 1) & 1) : (lc & 1);
                if (!warp_wait(&m->osc_full[lc & 1], (lc >> 1) & 1)) { fail(ERR_TIMEOUT_HANDOFF); break; }
                if (!warp_wait(&m->bar4[b], bph)) { fail(ERR_TIMEOUT_MMA); break; }
                tc_fence_after();
                const int *sx = m->osx[lc & 1];
                const float fq1 = exp2i(-sx[0]), fq2 = exp2i(-sx[1]);
                const float fp1 = exp2i(-sx[2]), fp2 = exp2i(-sx[3]);
                const int cc = c_begin + lc;
                const bool live = i < min(C, len - cc * C);
                uint4 *dst = reinterpret_cast<uint4 *>(o + ((size_t)(t0 + cc * C + i) * H + h) * D + dv0 + c0);
#pragma unroll
                for (int p = 0; p < K::kCU / 32; ++p) {
                    uint32_t x1[32], x4[32];
                    tmem_ld32(tmem + lane_off + K::TD1 + b * NB + c0 + p * 32, x1);
                    tmem_ld32(tmem + lane_off + K::TD4 + b * NB + c0 + p * 32, x4);
                    tmem_wait_ld();
                    if (live) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int j = q * 8 + 2 * e;
                                const float a = __uint_as_float(x1[j]) * fq1 * fq2 + __uint_as_float(x4[j]) * fp1 * fp2;
                                const float c2 = __uint_as_float(x1[j + 1]) * fq1 * fq2 + __uint_as_float(x4[j + 1]) * fp1 * fp2;
                                const __nv_bfloat162 b2 = __floats2bfloat162_rn(a, c2);
                                w[e] = *reinterpret_cast<const uint32_t *>(&b2);
                            }
                            dst[p * 4 + q] = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(&m->o_free[b]);
            }
        }
    } else if (warp == K::kIssuer) {
        // ======================================================= MMA issuer ====
        if (lane == 0) {
            // MN-major images: 8-row K groups 512 bytes apart, 16 K rows per MMA
            const uint64_t d_sb = sw64_mnmajor_desc(sbase + K::SB, 8192, 512);
            const uint64_t d_ub = sw64_mnmajor_desc(sbase + K::UB, 8192, 512);
            for (int lc = 0; lc < nl; ++lc) {
                if (*abort_flag) break;
                const uint32_t s = lc & 1, sph = (lc >> 1) & 1;
                const uint32_t b = K::kDB ? (lc & 1) : 0;                 // K̂/P stage = O buffer
                const uint32_t bph = K::kDB ? ((lc >> 1) & 1) : (lc & 1);
                // the buffers are normally ready long before the state block
                if (!mbar_wait_sleep(&m->full_a1[s], sph)) { fail(ERR_TIMEOUT_TMA); break; }
                const int prev = K::kDB ? lc - 2 : lc - 1;                // last user of O buffer b
                if (prev >= 0 && !mbar_wait_sleep(&m->o_free[b], K::kDB ? ((prev >> 1) & 1) : (prev & 1))) {
                    fail(ERR_TIMEOUT_HANDOFF);
                    break;
                }
                if (!mbar_wait_sleep(&m->s_ready, lc & 1)) { fail(ERR_TIMEOUT_HANDOFF); break; }
                tc_fence_after();
                const uint64_t d_a1 = sw128_kmajor_desc(sbase + K::A1 + s * 32768);
                // descriptors advance by (bytes >> 4) in their start-address field
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_f16_ss(tmem + K::TD1 + b * NB, d_a1 + (((k >> 2) * 16384 + (k & 3) * 32) >> 4),
                               d_sb + ((k * 1024) >> 4), K::IDESC, k != 0);
                mma_commit(&m->bar1);
                mma_commit(&m->empty_a1[s]);
                if (!mbar_wait_sleep(&m->full_kp[b], bph)) { fail(ERR_TIMEOUT_TMA); break; }
                if (!mbar_wait_sleep(&m->u_ready, lc & 1)) { fail(ERR_TIMEOUT_HANDOFF); break; }
                tc_fence_after();
                const uint64_t d_kh = sw128_kmajor_desc(sbase + K::KH + b * 16384);
                const uint64_t d_a4 = sw128_kmajor_desc(sbase + K::A4 + b * 16384);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_f16_ss(tmem + K::TD2, d_kh + ((k * 32) >> 4), d_ub + ((k * 1024) >> 4), K::IDESC, k != 0);
                mma_commit(&m->bar2);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_f16_ss(tmem + K::TD4 + b * NB, d_a4 + ((k * 32) >> 4), d_ub + ((k * 1024) >> 4), K::IDESC,
                               k != 0);
                mma_commit(&m->bar4[b]);
                mma_commit(&m->empty_kp[b]);
            }
        }
    } else if (lane == 0) {
        // ==================================================== record loader ====
        uint32_t issued[6] = {0, 0, 0, 0, 0, 0};
        uint64_t *bars[6] = {&m->full_a1[0], &m->full_a1[1], &m->full_u[0], &m->full_u[1],
                             &m->full_kp[0], &m->full_kp[1]};
        auto load_a1 = [&](int lc) {
            const int s = lc & 1;
            mbar_arrive_expect_tx(&m->full_a1[s], 32768);
            bulk_load(sm + K::A1 + s * 32768, rec_of(lc) + REC_A1, 32768, &m->full_a1[s]);
            ++issued[s];
        };
        auto load_u = [&](int lc) {   // this CTA's channel blocks of Ũ, and the exponents
            const int s = lc & 1;
            const uint8_t *r = rec_of(lc);
            mbar_arrive_expect_tx(&m->full_u[s], 256 * NB + 16);
            bulk_load(sm + K::UT + s * (256 * NB), r + REC_UT + part * (NB / 32) * 8192, 256 * NB,
                      &m->full_u[s]);
            bulk_load(m->ex[s], r + REC_EX, 16, &m->full_u[s]);
            ++issued[2 + s];
        };
        auto load_kp = [&](int lc) {
            const int b = K::kDB ? (lc & 1) : 0;
            const uint8_t *r = rec_of(lc);
            mbar_arrive_expect_tx(&m->full_kp[b], 16384 + 8192);
            bulk_load(sm + K::KH + b * 16384, r + REC_KH, 16384, &m->full_kp[b]);
            bulk_load(sm + K::A4 + b * 16384 + 8192, r + REC_PM, 8192, &m->full_kp[b]);
            ++issued[4 + b];
        };
        auto prefetch_rec = [&](int lc) {
            if (lc < nl) {
                const uint8_t *r = rec_of(lc);
#pragma unroll
                for (int q = 0; q < 5; ++q) bulk_prefetch_l2(r + q * 18128, 18128);
            }
        };
        constexpr int kKPAhead = K::kDB ? 2 : 1;   // K̂/P stages in flight
        load_a1(0);
        load_kp(0);
        load_u(0);
        if (nl > 1) {
            load_a1(1);
            load_u(1);
            if (K::kDB) load_kp(1);
        }
        prefetch_rec(1);
        prefetch_rec(2);
        // each buffer is refilled as soon as the step reading it has finished,
        // in the order those steps finish within a chunk
        for (int lc = 0; lc < nl; ++lc) {
            if (*abort_flag) break;
            const uint32_t s = lc & 1, sph = (lc >> 1) & 1;
            const uint32_t b = K::kDB ? (lc & 1) : 0;
            const uint32_t bph = K::kDB ? ((lc >> 1) & 1) : (lc & 1);
            if (!mbar_wait_sleep(&m->empty_a1[s], sph)) { fail(ERR_TIMEOUT_MMA); break; }
            if (lc + 2 < nl) load_a1(lc + 2);
            if (!mbar_wait_sleep(&m->empty_u[s], sph)) { fail(ERR_TIMEOUT_HANDOFF); break; }
            if (lc + 2 < nl) load_u(lc + 2);
            if (!mbar_wait_sleep(&m->empty_kp[b], bph)) { fail(ERR_TIMEOUT_MMA); break; }
            if (lc + kKPAhead < nl) load_kp(lc + kKPAhead);
            prefetch_rec(lc + 3);
        }
        // never leave a bulk copy in flight into this CTA's shared memory
        for (int q = 0; q < 6; ++q)
            if (issued[q] > 0) (void)mbar_wait_sleep(bars[q], (issued[q] - 1) & 1);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, K::TCOLS);
    }
}

// ------------------------------------------- chain kernel, transposed form ----
// One CTA per (sequence, head).  The products are written transposed so that
// the value channel n is the TMEM lane and the state-side operand is the A
// operand, read from TMEM as packed fp16:
//
//   M1  D1^T = S_h [-W; Q̃]^T      (A = S fp16 in TMEM, B = the record's [-W; Q̃])
//                                  columns 0-63: X^T, 64-127: inter-chunk output
//   M2  ΔS   = U^T_h K̂            (A = U^T fp16 in TMEM, B = the record's K̂^T)
//   M4  O4^T = U^T_h (P ⊙ causal)^T   (B = the record's P)
//
// Each row of an fp16 A operand (one value channel) carries its own
// power-of-two scale, so the threads that share a row only exchange one
// value; there are no shared-memory operand writes.  4 kRQ row warps (warp
// w: lanes of sub-partition w % 4, part w / 4 of each row) run U, the state
// update and the output, meeting at one barrier per step that also carries
// the decision to stop; the next warp issues the MMAs, the last one loads the
// records.  The output tile goes through shared memory so that it leaves in
// 16-byte row segments.
// TMEM loads / stores of N consecutive columns (N = 8, 16 or 32), as many
// calls as needed for larger N.
template <int N>
__device__ __forceinline__ void tmem_ldn(uint32_t taddr, uint32_t (&r)[N]) {
    if constexpr (N == 16) {
        tmem_ld16(taddr, r);
    } else {
        static_assert(N % 32 == 0, "column count");
#pragma unroll
        for (int p = 0; p < N / 32; ++p) tmem_ld32(taddr + p * 32, *reinterpret_cast<uint32_t (*)[32]>(r + p * 32));
    }
}
template <int N>
__device__ __forceinline__ void tmem_stn(uint32_t taddr, const uint32_t (&r)[N]) {
    if constexpr (N == 8) {
        tmem_st8(taddr, r);
    } else if constexpr (N == 16) {
        tmem_st16(taddr, r);
    } else {
        static_assert(N % 32 == 0, "column count");
#pragma unroll
        for (int p = 0; p < N / 32; ++p)
            tmem_st32(taddr + p * 32, *reinterpret_cast<const uint32_t (*)[32]>(r + p * 32));
    }
}

constexpr int kRQ = 2;                     // threads per row (value channel)
constexpr int kRowWarps = 4 * kRQ;
constexpr int kRowThreads = 32 * kRowWarps;
constexpr int kSC = D / kRQ;               // state columns per thread
constexpr int kTK = C / kRQ;               // tokens per thread (U and output)
constexpr int kTThreads = kRowThreads + 64;
constexpr uint32_t TO_A1 = 0;          // [-W; Q̃] fp16 images, 2 stages of 32 KiB
constexpr uint32_t TO_KH = 65536;      // K̂^T fp16, 2 stages of 16 KiB
constexpr uint32_t TO_PM = 98304;      // P fp16, 2 stages of 8 KiB
constexpr uint32_t TO_UT = 114688;     // Ũ fp32, 2 stages of 32 KiB
constexpr uint32_t TO_OS = 180224;     // output tile [64 tok][128 ch] bf16, 2 buffers of 16 KiB
constexpr uint32_t TO_MISC = 212992;
constexpr uint32_t TSMEM = TO_MISC + 12288;
constexpr uint32_t TT_D1 = 0, TT_DS = 128, TT_O4 = 256, TT_SA = 320, TT_UA = 384, TT_COLS = 512;
constexpr uint32_t IDESC_H128 = make_idesc(0, 128, 128), IDESC_H64 = make_idesc(0, 128, 64);

struct TMisc {
    uint64_t full_a1[2], full_u[2], full_kp[2];
    uint64_t empty_a1[2], empty_u[2], empty_kp[2];
    uint64_t bar1, bar2, bar4;
    uint64_t u_ready, s_ready;
    uint32_t tmem_base;
    int abort_flag;
    alignas(16) int ex[2][4];      // record exponents {s_W, s_Q, s_K, s_P}, with the Ũ stage
    alignas(16) float gam[2][D];   // exp(G_C), with the Ũ stage
    float xu[2][kRQ * D], xs[2][kRQ * D];   // part-row maxima exchanged between a row's threads
};
static_assert(sizeof(TMisc) <= 12288 && TSMEM <= 232448, "chain smem overflow");

template <bool CHANNEL>
__global__ void __launch_bounds__(kTThreads, 1)
chain_t_kernel(const uint8_t *__restrict__ recs, const float *h0, float *fin, float *ws_state,
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
    const int sub = warp & 3, qp = (warp >> 2) % kRQ;   // TMEM sub-partition, row quarter
    const int row = sub * 32 + lane;                     // value channel = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
    const size_t sg = (((size_t)n * H + h) * D + row) * D + qp * kSC;

    if (nl == 0) {   // empty sequence: the state passes through
        if (s_out != nullptr && warp < kRowWarps) {
#pragma unroll
            for (int j = 0; j < kSC; j += 4) {
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                if (s_in != nullptr) x = *reinterpret_cast<const float4 *>(s_in + sg + j);
                *reinterpret_cast<float4 *>(s_out + sg + j) = x;
            }
        }
        return;
    }
    if ((sbase & 1023u) != 0) {
        if (tid == 0) atomicOr(err, ERR_SMEM_ALIGN);
        return;
    }
    uint8_t *sm = smem_raw;
    TMisc *m = reinterpret_cast<TMisc *>(sm + TO_MISC);
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&m->full_a1[s], 1);
            mbar_init(&m->full_u[s], 1);
            mbar_init(&m->full_kp[s], 1);
            mbar_init(&m->empty_a1[s], 1);
            mbar_init(&m->empty_u[s], kRowThreads);
            mbar_init(&m->empty_kp[s], 1);
        }
        mbar_init(&m->bar1, 1);
        mbar_init(&m->bar2, 1);
        mbar_init(&m->bar4, 1);
        mbar_init(&m->u_ready, kRowThreads);
        mbar_init(&m->s_ready, kRowThreads);
        m->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&m->tmem_base, TT_COLS);
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

    if (warp < kRowWarps) {
        // ============================= row warps: channel `row`, quarter `qp` ====
        bool stop = false;
        // Barrier over the row warps; every row warp passes the same sequence of
        // them, and `stop` leaves it the same in all threads.
        auto rows_sync = [&]() { stop = named_sync_or(1, kRowThreads, stop || *abort_flag != 0); };
        // the row's largest |value| over its kRQ parts
        auto row_max = [&](float mx, float *slots) {
            slots[qp * D + row] = mx;
            rows_sync();
#pragma unroll
            for (int k = 0; k < kRQ; ++k) mx = fmaxf(mx, slots[k * D + row]);
            return mx;
        };
        float S[kSC];
#pragma unroll
        for (int j = 0; j < kSC; j += 4) {
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (s_in != nullptr) x = *reinterpret_cast<const float4 *>(s_in + sg + j);
            S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
        }
        // fp16 copy of the state row (A of M1) with the row's own scale
        auto publish = [&](int lc) {
            float mx = 0.f;
#pragma unroll
            for (int j = 0; j < kSC; ++j) mx = fmaxf(mx, fabsf(S[j]));
            const int sS = scale_exp(row_max(mx, m->xs[lc & 1]));
            const float f = exp2i(sS);
            uint32_t w[kSC / 2];
#pragma unroll
            for (int j = 0; j < kSC / 2; ++j) w[j] = f2h2_bits(S[2 * j] * f, S[2 * j + 1] * f);
            tmem_stn<kSC / 2>(tmem + lane_off + TT_SA + qp * (kSC / 2), w);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&m->s_ready);
            return sS;
        };
        int sS = publish(0);
        for (int lc = 0; lc < nl && !stop; ++lc) {
            const uint32_t s = lc & 1, sph = (lc >> 1) & 1;
            // (a) D1^T: X^T and the inter-chunk output of this thread's tokens
            if (!warp_wait(&m->bar1, lc & 1)) { fail(ERR_TIMEOUT_MMA); stop = true; }
            if (!stop && !warp_wait(&m->full_u[s], sph)) { fail(ERR_TIMEOUT_TMA); stop = true; }
            uint32_t x[kTK], oi[kTK];
            int sW = 0, sQ = 0, sK = 0, sP = 0;
            float mx = 0.f;
            if (!stop) {
                tc_fence_after();
                tmem_ldn<kTK>(tmem + lane_off + TT_D1 + qp * kTK, x);
                tmem_ldn<kTK>(tmem + lane_off + TT_D1 + 64 + qp * kTK, oi);
                sW = m->ex[s][0]; sQ = m->ex[s][1]; sK = m->ex[s][2]; sP = m->ex[s][3];
                const float fa = exp2i(-sW), fb = exp2i(-sS);
                const uint8_t *ut = sm + TO_UT + s * 32768 - REC_UT;
                tmem_wait_ld();
#pragma unroll
                for (int jj = 0; jj < kTK; ++jj) {
                    const float u = *reinterpret_cast<const float *>(ut + rec_ut_offset(qp * kTK + jj, row)) +
                                    __uint_as_float(x[jj]) * fa * fb;
                    x[jj] = __float_as_uint(u);
                    mx = fmaxf(mx, fabsf(u));
                }
            }
            const int sU = scale_exp(row_max(mx, m->xu[lc & 1]));
            if (stop) break;
            {   // U^T row part (A of M2 and M4): kTK tokens = kTK / 2 packed columns
                const float f = exp2i(sU);
                uint32_t w[kTK / 2];
#pragma unroll
                for (int j = 0; j < kTK / 2; ++j)
                    w[j] = f2h2_bits(__uint_as_float(x[2 * j]) * f, __uint_as_float(x[2 * j + 1]) * f);
                tmem_stn<kTK / 2>(tmem + lane_off + TT_UA + qp * (kTK / 2), w);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&m->u_ready);
            }
            // (b) S = S Diag(exp(G_C)) + ΔS
            if (!warp_wait(&m->bar2, lc & 1)) { fail(ERR_TIMEOUT_MMA); stop = true; }
            if (!stop) {
                tc_fence_after();
                const float f1 = exp2i(-sK), f2 = exp2i(-sU);
                const float *gam = m->gam[s] + qp * kSC;
                uint32_t d[kSC];
                tmem_ldn<kSC>(tmem + lane_off + TT_DS + qp * kSC, d);
                tmem_wait_ld();
#pragma unroll
                for (int jj = 0; jj < kSC; ++jj) {
                    const float gc = CHANNEL ? gam[jj] : m->gam[s][0];
                    S[jj] = fmaf(gc, S[jj], __uint_as_float(d[jj]) * f1 * f2);
                }
                tc_fence_before();
                mbar_arrive(&m->empty_u[s]);   // Ũ, exponents and gate of this stage are read
            }
            // (stop may differ between warps here; the barrier in (c) settles it)
            const int sS_next = (lc + 1 < nl) ? publish(lc + 1) : 0;
            // (c) output rows: O^T = O_inter^T + O4^T, unscaled, for this thread's
            //     tokens, staged as a [token][channel] tile
            if (!warp_wait(&m->bar4, lc & 1)) { fail(ERR_TIMEOUT_MMA); stop = true; }
            if (!stop) {
                uint32_t o4[kTK];
                tc_fence_after();
                tmem_ldn<kTK>(tmem + lane_off + TT_O4 + qp * kTK, o4);
                tmem_wait_ld();
                const float fq1 = exp2i(-sQ), fq2 = exp2i(-sS), fp1 = exp2i(-sP), fp2 = exp2i(-sU);
                const uint32_t stile = sbase + TO_OS + s * 16384 + qp * kTK * 256 + row * 2;
#pragma unroll
                for (int jj = 0; jj < kTK; ++jj) {
                    const __nv_bfloat16 b = __float2bfloat16_rn(__uint_as_float(oi[jj]) * fq1 * fq2 +
                                                                __uint_as_float(o4[jj]) * fp1 * fp2);
                    st_shared_b16(stile + jj * 256, *reinterpret_cast<const uint16_t *>(&b));
                }
            }
            rows_sync();
            if (stop) break;
            {   // 64 rows x 256 bytes leave as 16-byte segments; rows past the end stay
                const int cc = c_begin + lc;
                const int cl = min(C, len - cc * C);
                const uint32_t tile = sbase + TO_OS + s * 16384;
#pragma unroll
                for (int q = 0; q < 1024 / kRowThreads; ++q) {
                    const int e = q * kRowThreads + tid;   // segment: row e / 16, 16 bytes e % 16
                    const int i = e >> 4, seg = e & 15;
                    if (i < cl) {
                        const uint4 v = ld_shared_v4(tile + i * 256 + seg * 16);
                        *reinterpret_cast<uint4 *>(o + ((size_t)(t0 + cc * C + i) * H + h) * D + seg * 8) = v;
                    }
                }
            }
            sS = sS_next;
        }
        if (s_out != nullptr) {
#pragma unroll
            for (int j = 0; j < kSC; j += 4)
                *reinterpret_cast<float4 *>(s_out + sg + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    } else if (warp == kRowWarps) {
        // ======================================================= MMA issuer ====
        if (lane == 0) {
            for (int lc = 0; lc < nl; ++lc) {
                if (*abort_flag) break;
                const uint32_t s = lc & 1, sph = (lc >> 1) & 1;
                if (!mbar_wait_sleep(&m->full_a1[s], sph)) { fail(ERR_TIMEOUT_TMA); break; }
                if (!mbar_wait_sleep(&m->s_ready, lc & 1)) { fail(ERR_TIMEOUT_HANDOFF); break; }
                tc_fence_after();
                const uint64_t d_a1 = sw128_kmajor_desc(sbase + TO_A1 + s * 32768);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_f16_ts(tmem + TT_D1, tmem + TT_SA + k * 8,
                               d_a1 + (((k >> 2) * 16384 + (k & 3) * 32) >> 4), IDESC_H128, k != 0);
                mma_commit(&m->bar1);
                mma_commit(&m->empty_a1[s]);
                if (!mbar_wait_sleep(&m->full_kp[s], sph)) { fail(ERR_TIMEOUT_TMA); break; }
                if (!mbar_wait_sleep(&m->u_ready, lc & 1)) { fail(ERR_TIMEOUT_HANDOFF); break; }
                tc_fence_after();
                const uint64_t d_kh = sw128_kmajor_desc(sbase + TO_KH + s * 16384);
                const uint64_t d_pm = sw128_kmajor_desc(sbase + TO_PM + s * 8192);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_f16_ts(tmem + TT_DS, tmem + TT_UA + k * 8, d_kh + ((k * 32) >> 4), IDESC_H128, k != 0);
                mma_commit(&m->bar2);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_f16_ts(tmem + TT_O4, tmem + TT_UA + k * 8, d_pm + ((k * 32) >> 4), IDESC_H64, k != 0);
                mma_commit(&m->bar4);
                mma_commit(&m->empty_kp[s]);
            }
        }
    } else if (lane == 0) {
        // ==================================================== record loader ====
        const uint32_t gbytes = CHANNEL ? 512u : 16u;
        uint32_t issued[6] = {0, 0, 0, 0, 0, 0};
        uint64_t *bars[6] = {&m->full_a1[0], &m->full_a1[1], &m->full_u[0], &m->full_u[1],
                             &m->full_kp[0], &m->full_kp[1]};
        auto load_a1 = [&](int lc) {
            const int s = lc & 1;
            mbar_arrive_expect_tx(&m->full_a1[s], 32768);
            bulk_load(sm + TO_A1 + s * 32768, rec_of(lc) + REC_A1, 32768, &m->full_a1[s]);
            ++issued[s];
        };
        auto load_u = [&](int lc) {
            const int s = lc & 1;
            const uint8_t *r = rec_of(lc);
            mbar_arrive_expect_tx(&m->full_u[s], 32768 + 16 + gbytes);
            bulk_load(sm + TO_UT + s * 32768, r + REC_UT, 32768, &m->full_u[s]);
            bulk_load(m->ex[s], r + REC_EX, 16, &m->full_u[s]);
            bulk_load(m->gam[s], r + REC_GC, gbytes, &m->full_u[s]);
            ++issued[2 + s];
        };
        auto load_kp = [&](int lc) {
            const int s = lc & 1;
            const uint8_t *r = rec_of(lc);
            mbar_arrive_expect_tx(&m->full_kp[s], 16384 + 8192);
            bulk_load(sm + TO_KH + s * 16384, r + REC_KH, 16384, &m->full_kp[s]);
            bulk_load(sm + TO_PM + s * 8192, r + REC_PM, 8192, &m->full_kp[s]);
            ++issued[4 + s];
        };
        auto prefetch_rec = [&](int lc) {
            if (lc < nl) {
                const uint8_t *r = rec_of(lc);
#pragma unroll
                for (int q = 0; q < 5; ++q) bulk_prefetch_l2(r + q * 18128, 18128);
            }
        };
        load_a1(0);
        load_kp(0);
        load_u(0);
        if (nl > 1) {
            load_a1(1);
            load_u(1);
            load_kp(1);
        }
        prefetch_rec(2);
        prefetch_rec(3);
        for (int lc = 0; lc < nl; ++lc) {
            if (*abort_flag) break;
            const uint32_t s = lc & 1, sph = (lc >> 1) & 1;
            if (!mbar_wait_sleep(&m->empty_a1[s], sph)) { fail(ERR_TIMEOUT_MMA); break; }
            if (lc + 2 < nl) load_a1(lc + 2);
            if (!mbar_wait_sleep(&m->empty_kp[s], sph)) { fail(ERR_TIMEOUT_MMA); break; }
            if (lc + 2 < nl) load_kp(lc + 2);
            if (!mbar_wait_sleep(&m->empty_u[s], sph)) { fail(ERR_TIMEOUT_HANDOFF); break; }
            if (lc + 2 < nl) load_u(lc + 2);
            prefetch_rec(lc + 4);
        }
        // never leave a bulk copy in flight into this CTA's shared memory
        for (int q = 0; q < 6; ++q)
            if (issued[q] > 0) (void)mbar_wait_sleep(bars[q], (issued[q] - 1) & 1);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TT_COLS);
    }
}

// ------------------------------------------------------------------ host ----

constexpr size_t kHeaderBytes = 256;                        // error word
constexpr size_t kMaxRecordBytes = size_t(1) << 30;         // records per window
// Up to 64 chains the two kernels beat the single-kernel plan: its chunk
// period is set by the chunk-local work, which the prep kernel spreads over
// all SMs.  With more chains that plan already keeps most SMs busy and the
// prep kernel's extra record traffic no longer pays (measured on B200).
constexpr int kSplitMaxChains = 64;

struct SplitPlan {
    int chains = 0, max_chunks = 0, window = 0, windows = 0;
    int pieces = 1;   // pipeline pieces of a single window (prep of piece k + 1 beside chain k)
    size_t state_off = 0, rec_off = 0, bytes = 0;
};

// Pipeline pieces of one window: the prep kernel of piece k + 1 runs beside
// the chain kernel of piece k, and on the SMs the chain leaves free a chunk's
// prep takes about 3/4 of a chunk's chain step, so each piece may be 1.3 times
// the one before: 12, 16, 21, 27, 35, ... chunks, the last one the remainder.
// Writes the piece boundaries (count + 1 of them) and returns the count.
constexpr int kMaxPieces = 32;
int piece_schedule(int max_chunks, int *bounds) {
    int n = 0, c = 0, size = 12;
    bounds[0] = 0;
    while (c < max_chunks && n < kMaxPieces) {
        c = (n + 1 == kMaxPieces) ? max_chunks : std::min(c + size, max_chunks);
        bounds[++n] = c;
        size = (size * 13 + 9) / 10;
    }
    return n;
}

// With equal lengths (no cu_seqlens) every sequence has total_T / num_seqs
// tokens; otherwise the lengths live on the device and total_T bounds them.
// The equal-length plan never needs more workspace than the general one (its
// window is no larger, and it needs the state area only when that one does).
bool make_split_plan(int num_seqs, int total_T, int H, SplitPlan &p, bool equal_lengths = false) {
    const long long chains = (long long)num_seqs * H;
    if (chains < 1 || chains > kSplitMaxChains || total_T <= 0) return false;
    p.chains = (int)chains;
    const int longest = equal_lengths ? total_T / num_seqs : total_T;
    p.max_chunks = (longest + C - 1) / C;   // no sequence has more chunks
    const size_t per = (size_t)p.chains * REC_BYTES;
    const size_t fit = kMaxRecordBytes / per;
    p.window = (int)(fit < 1 ? 1 : (fit < (size_t)p.max_chunks ? fit : (size_t)p.max_chunks));
    p.windows = (p.max_chunks + p.window - 1) / p.window;
    int bounds[kMaxPieces + 1];
    p.pieces = p.windows == 1 ? piece_schedule(p.max_chunks, bounds) : 1;
    const size_t state =
        (p.windows > 1 || p.pieces > 1) ? (size_t)p.chains * D * D * sizeof(float) : 0;
    p.state_off = kHeaderBytes;
    p.rec_off = (kHeaderBytes + state + 1023) & ~size_t(1023);
    p.bytes = p.rec_off + (size_t)p.window * per;
    return true;
}


// Per-device helper streams for the pipelined plan: chain kernels on a
// high-priority stream, prep kernels on a low-priority one, forked from and
// joined back into the caller's stream with events (capturable in a graph).
struct Helpers {
    bool ready = false;
    cudaStream_t chain_s = nullptr, prep_s = nullptr;
    cudaEvent_t fork = nullptr, prep_done = nullptr, join = nullptr;
};
constexpr int kMaxDevices = 64;
std::mutex g_helpers_mutex;
Helpers g_helpers[kMaxDevices];

cudaError_t get_helpers(Helpers **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    Helpers &hs = g_helpers[dev];
    if (!hs.ready) {
        int least = 0, greatest = 0;
        e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
        if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&hs.chain_s, cudaStreamNonBlocking, greatest);
        if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&hs.prep_s, cudaStreamNonBlocking, least);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hs.fork, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hs.prep_done, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hs.join, cudaEventDisableTiming);
        if (e != cudaSuccess) return e;
        hs.ready = true;
    }
    *out = &hs;
    return cudaSuccess;
}

template <int NB>
cudaError_t launch_chain(bool channel, int chains, const uint8_t *recs, const float *h0, float *fin,
                         float *state, const int32_t *cu, int num_seqs, int total_T, int H, int c0,
                         int c1, __nv_bfloat16 *o, uint32_t *err, cudaStream_t stream) {
    using K = Chain<NB>;
    auto kern = channel ? chain_kernel<true, NB> : chain_kernel<false, NB>;
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void *>(kern), (int)K::SMEM);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(chains * (D / NB)), K::kThreads, K::SMEM, stream>>>(
        recs, h0, fin, state, cu, num_seqs, total_T, H, c0, c1, o, err);
    return cudaGetLastError();
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
    if (!make_split_plan(num_seqs, total_T, H, p, cu == nullptr)) return cudaErrorInvalidValue;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint32_t *err = reinterpret_cast<uint32_t *>(ws);
    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(uint32_t), stream);
    if (e != cudaSuccess) return e;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, total_T, Hqk) || !make_map(&mk, k, total_T, Hqk) ||
        !make_map(&mv, v, total_T, H))
        return cudaErrorInvalidValue;
    auto prep = channel ? prep_kernel<true> : prep_kernel<false>;
    e = ensure_dynamic_smem(reinterpret_cast<const void *>(prep), (int)PREP_SMEM);
    if (e != cudaSuccess) return e;
    float *state = (p.windows > 1 || p.pieces > 1) ? reinterpret_cast<float *>(ws + p.state_off) : nullptr;
    uint8_t *recs = ws + p.rec_off;
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(o);
    // Few chains: split d_v over four CTAs each (NB = 32), so that more SMs
    // share the chain work; otherwise one CTA per chain, transposed form.
    const bool dv_split = p.chains * 4 <= 148;
    auto chain_t = channel ? chain_t_kernel<true> : chain_t_kernel<false>;
    e = ensure_dynamic_smem(reinterpret_cast<const void *>(chain_t), (int)TSMEM);
    if (e != cudaSuccess) return e;
    auto run_chain = [&](int c0, int c1, const uint8_t *r, cudaStream_t st) {
        if (dv_split)
            return launch_chain<32>(channel, p.chains, r, h0, fin, state, cu, num_seqs, total_T, H, c0, c1,
                                    out, err, st);
        chain_t<<<(unsigned)p.chains, kTThreads, TSMEM, st>>>(r, h0, fin, state, cu, num_seqs, total_T, H,
                                                                c0, c1, out, err);
        return cudaGetLastError();
    };
    auto run_prep = [&](int c0, int c1, uint8_t *r, cudaStream_t st) {
        prep<<<dim3((unsigned)(c1 - c0), (unsigned)p.chains), kPrepThreads, PREP_SMEM, st>>>(
            mq, mk, mv, g, beta, cu, num_seqs, total_T, Hqk, H, c0, r, err);
        return cudaGetLastError();
    };
    if (p.pieces > 1) {
        // every record has its own slot: the prep kernel of piece k + 1 runs on
        // the SMs the chain kernel of piece k leaves free
        std::lock_guard<std::mutex> lock(g_helpers_mutex);
        Helpers *hs = nullptr;
        e = get_helpers(&hs);
        if (e != cudaSuccess) return e;
        int bounds[kMaxPieces + 1];
        piece_schedule(p.max_chunks, bounds);
        e = cudaEventRecord(hs->fork, stream);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(hs->prep_s, hs->fork, 0);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(hs->chain_s, hs->fork, 0);
        for (int k = 0; k < p.pieces && e == cudaSuccess; ++k) {
            const int c0 = bounds[k], c1 = bounds[k + 1];
            uint8_t *r = recs + (size_t)c0 * p.chains * REC_BYTES;
            e = run_prep(c0, c1, r, hs->prep_s);
            if (e == cudaSuccess) e = cudaEventRecord(hs->prep_done, hs->prep_s);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(hs->chain_s, hs->prep_done, 0);
            if (e == cudaSuccess) e = run_chain(c0, c1, r, hs->chain_s);
        }
        if (e == cudaSuccess) e = cudaEventRecord(hs->join, hs->chain_s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, hs->join, 0);
        return e;
    }
    for (int w = 0; w < p.windows; ++w) {
        const int c0 = w * p.window;
        const int c1 = c0 + p.window < p.max_chunks ? c0 + p.window : p.max_chunks;
        e = run_prep(c0, c1, recs, stream);
        if (e != cudaSuccess) return e;
        e = run_chain(c0, c1, recs, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace gdr
