// Chunked prefill of the gated delta rule on the sm_100a tensor cores
// (tcgen05 MMA with TMEM accumulators, operands staged by TMA), bf16 I/O,
// d_k = d_v = 128, scalar gate (Gated DeltaNet) or per-key-channel gate
// (Kimi Delta Attention).
//
// The algebra is the exact chunk rearrangement of the recurrence on the page
// "How the New Flash Models Work: Inside GLM-5.3-Flash and Qwen3.8-Flash-Next"
// (section "Linear attention: a fixed-size memory in place of the cache",
// Gated DeltaNet and Kimi Delta Attention equations).  For a chunk of C = 64
// tokens entering with state S (d_v x d_k), within-chunk cumulative log-gate
// G_i (a scalar, or one value per key channel) and Γ_i = exp(G_i):
//
//   A_ij = β_i k_i^T Diag(exp(G_i - G_j)) k_j  (j < i),   T = (I + A)^-1
//   W    = T diag(β) (K ⊙ Γ),   Ũ = T diag(β) V
//   U    = Ũ - W S^T                                (corrected values)
//   O    = (Q ⊙ Γ) S^T + (P ⊙ causal) U,  P_ij = q_i^T Diag(exp(G_i - G_j)) k_j
//   S'   = S Diag(Γ_C) + U^T K̂,   K̂_j = k_j ⊙ exp(G_C - G_j)
//
// Every exponent in these formulas is <= 0.  The MMAs are written transposed
// so that the 128-wide d_v / d_k dimension is the M = 128 dimension (TMEM
// lane = matrix row):
//
//   P1  [K;Q] K^T  M=128 N=64  -> rows 0-63 give A (with β and decay),
//                                 rows 64-127 give P
//   P2  W^T = K'^T T^T, Ũ^T = V'^T T^T           (tf32)
//   S1  U^T += S (-W)^T       S1'  O^T = S Q̃^T    (tf32, A = S from TMEM)
//   S3  ΔS = U^T K̂            S2   O^T += U^T P^T (tf32, A = U from TMEM)
//
// Gated DeltaNet runs P1 on the exact bf16 inputs and applies the scalar
// decays afterwards in fp32.  Kimi Delta Attention folds the per-channel
// decays into the operands around a mid-chunk reference R (token 31):
// [K ⊙ e^{G-R}; Q ⊙ e^{G-R}] (K ⊙ e^{R-G})^T, in fp16 (11-bit significand,
// as precise as tf32 at half the footprint).  A chunk whose scaled operands
// would leave fp16's range instead computes A and P exactly on CUDA cores.
//
// Operands that feed the state are tf32, rounded to nearest: bf16 would put
// ~2^-9 relative error into every chunk's update.  The fp32 master state
// lives in registers (thread = row of S, 64 columns); a tf32 copy in TMEM is
// the A operand of S1/S1'.
//
// One CTA of 16 warps per (sequence, head), split into two groups that run
// one chunk apart:
//   * the chain group (warps 0-7) owns the state and runs only the
//     state-dependent steps S1/S1', the rounding of U, S3/S2, the state
//     update and the output store;
//   * the prep group (warps 8-15) runs every chunk-local step for the next
//     chunk: TMA loads, gates, P1, A and P, the 64 x 64 unit-triangular
//     inverse (blocked 16 x 16 forward substitution), the tf32 operands, P2
//     and -W.
// They hand off through mbarriers; Ũ (TMEM) and P (shared memory) are
// double-buffered so the prep of chunk c+1 overlaps the chain of chunk c.
// Rows past a sequence's end get β = 0 and g = 0, which makes their A rows,
// u and gate increments vanish.  Every mbarrier wait is bounded; on timeout
// the CTA records an error bit in the workspace word and stops.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

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

constexpr int kThreads = 512;

// Shared-memory map (byte offsets from the 1024-aligned dynamic base).
constexpr uint32_t OFF_KQ = 0;        // bf16 tiles [K d0-63][Q d0-63][K d64-127][Q d64-127], 8 KiB each
constexpr uint32_t OFF_V = 32768;     // bf16 tiles [V d0-63][V d64-127]
constexpr uint32_t OFF_X1 = 49152;    // K'^T [dk][tok] tf32, then -W [tok][dk] tf32
constexpr uint32_t OFF_X2 = 81920;    // scratch (A, T fp32 / KDA fp16 P1 operand / G), then V'^T
constexpr uint32_t OFF_KH = 114688;   // K̂^T [dk][tok] tf32
constexpr uint32_t OFF_QT = 147456;   // Q̃ [tok][dk] tf32
constexpr uint32_t OFF_PM = 180224;   // P [i][j] tf32, two slots of 16 KiB
constexpr uint32_t OFF_TM = 212992;   // T [i][j] tf32 (scratch before that)
constexpr uint32_t OFF_MISC = 229376;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 3072;   // 232448: the per-block maximum

// TMEM columns.
constexpr uint32_t TM_P1W = 0, TM_U0 = 64, TM_O = 192, TM_DS = 256, TM_S = 384;
constexpr uint32_t TMEM_COLS = 512;


constexpr uint32_t ERR_TIMEOUT_TMA = 1u, ERR_TIMEOUT_MMA = 2u, ERR_TIMEOUT_HANDOFF = 4u,
                   ERR_SMEM_ALIGN = 8u;

struct Misc {
    uint64_t bar_tma, bar_p, bar_ready, bar_s1, bar_s3;
    uint32_t tmem_base;
    int abort_flag;
    int slow;
    int wide;                          // Gated DeltaNet: chunk decay beyond e^-80
    union alignas(16) {
        struct {                       // Gated DeltaNet, per chunk (prep only)
            float beta[C], G[C], gam[C], kp[C], kh[C], ieg[C];
        } s;
        struct {                       // Kimi Delta Attention, per chunk (prep only)
            float beta[C], T0[D], T1[D];
        } c;
    } u;                               // beta comes first in both layouts
    alignas(16) float gcb[2][D];       // exp(G_C) handed to the chain, per chunk slot
};
static_assert(sizeof(Misc) <= 3072, "misc area overflow");
// float4 reads of the per-token arrays need 16-byte alignment
static_assert(offsetof(Misc, u) % 16 == 0 && (C * 4) % 16 == 0, "misc arrays misaligned");

// Bounded wait inside one group; all threads of the group agree on stopping.
__device__ __forceinline__ bool group_wait(uint64_t *bar, uint32_t phase, Misc *m, uint32_t *err,
                                           uint32_t code, int gid) {
    const bool ok = mbar_wait(bar, phase);
    if (!ok) {
        m->abort_flag = 1;
        atomicOr(err, code);
    }
    group_sync(gid);
    return m->abort_flag == 0;
}

template <bool CHANNEL>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const float *__restrict__ g,
                  const float *__restrict__ beta, const float *h0,
                  const int32_t *__restrict__ cu, int num_seqs, int total_T, int Hqk, int H,
                  __nv_bfloat16 *__restrict__ o, float *fin, uint32_t *err) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = smem_u32(smem_raw);
    if ((sbase & 1023u) != 0) {
        if (threadIdx.x == 0) atomicOr(err, ERR_SMEM_ALIGN);
        return;
    }
    uint8_t *sm = smem_raw;
    Misc *m = reinterpret_cast<Misc *>(sm + OFF_MISC);

    const int h = blockIdx.x % H;          // value head
    const int n = blockIdx.x / H;
    const int hq = h / (H / Hqk);          // its query/key head
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int sub = warp & 3;           // TMEM sub-partition of this warp
    const int half = (warp >> 2) & 1;   // column half handled inside the group
    const int row = sub * 32 + lane;    // TMEM lane = matrix row
    const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;

    if (tid == 0) {
        mbar_init(&m->bar_tma, 1);
        mbar_init(&m->bar_p, 1);
        mbar_init(&m->bar_ready, 1);
        mbar_init(&m->bar_s1, 1);
        mbar_init(&m->bar_s3, 1);
        m->abort_flag = 0;
        m->slow = 0;
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
    const int nchunks = (len + C - 1) / C;

    if (tid < 256) {
        // ===================================================== chain group ====
        const size_t sg = (((size_t)n * H + h) * D + row) * D + half * 64;
        float S[64];
#pragma unroll
        for (int j = 0; j < 64; j += 4) {
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (h0 != nullptr) x = *reinterpret_cast<const float4 *>(h0 + sg + j);
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
        group_sync(1);

        // output epilogue of a finished chunk: lane = value channel, columns = tokens
        auto store_o = [&](int cc) {
            const int tok0 = t0 + cc * C;
            const int cl = min(C, len - cc * C);
            uint32_t x[32];
            tmem_ld32(tmem + lane_off + TM_O + half * 32, x);
            tmem_wait_ld();
#pragma unroll
            for (int ii = 0; ii < 32; ++ii) {
                const int i = half * 32 + ii;
                if (i < cl)
                    o[((size_t)(tok0 + i) * H + h) * D + row] =
                        __float2bfloat16_rn(__uint_as_float(x[ii]));
            }
        };
        bool done_ok = true;
        for (int c = 0; c < nchunks; ++c) {
            const uint32_t par = c & 1;
            const uint32_t tmU = TM_U0 + par * 64;
            if (!group_wait(&m->bar_ready, par, m, err, ERR_TIMEOUT_HANDOFF, 1)) { done_ok = false; break; }
            tc_fence_after();
            // S1: U^T += S (-W)^T -- the only product on the state's critical path
            if (tid == 0) {
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const uint32_t off = (k >> 2) * 8192 + (k & 3) * 32;
                    mma_tf32_ts(tmem + tmU, tmem + TM_S + k * 8,
                                sw128_kmajor_desc(sbase + OFF_X1 + off), IDESC_N64, 1);
                }
                mma_commit(&m->bar_s1);
            }
            if (c >= 1) store_o(c - 1);   // overlaps S1
            if (!group_wait(&m->bar_s1, par, m, err, ERR_TIMEOUT_MMA, 1)) { done_ok = false; break; }
            tc_fence_after();
            {   // round U to tf32 in place: it is the A operand of S3 and S2
                uint32_t x[32];
                tmem_ld32(tmem + lane_off + tmU + half * 32, x);
                tmem_wait_ld();
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) x[jj] = to_tf32(__uint_as_float(x[jj]));
                tmem_st32(tmem + lane_off + tmU + half * 32, x);
                tmem_wait_st();
            }
            tc_fence_before();
            group_sync(1);
            if (tid == 0) {
                tc_fence_after();
                // S3: ΔS = U^T K̂ (state) first, then the output products
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t kb = k >> 2, kk = k & 3;
                    mma_tf32_ts(tmem + TM_DS, tmem + tmU + k * 8,
                                sw128_kmajor_desc(sbase + OFF_KH + kb * 16384 + kk * 32),
                                IDESC_N128, k != 0);
                }
                // S1': O^T = S Q̃^T ; S2: O^T += U^T (P⊙causal)^T
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const uint32_t off = (k >> 2) * 8192 + (k & 3) * 32;
                    mma_tf32_ts(tmem + TM_O, tmem + TM_S + k * 8,
                                sw128_kmajor_desc(sbase + OFF_QT + off), IDESC_N64, k != 0);
                }
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t kb = k >> 2, kk = k & 3;
                    mma_tf32_ts(tmem + TM_O, tmem + tmU + k * 8,
                                sw128_kmajor_desc(sbase + OFF_PM + par * 16384 + kb * 8192 + kk * 32),
                                IDESC_N64, 1);
                }
                mma_commit(&m->bar_s3);
            }
            if (!group_wait(&m->bar_s3, par, m, err, ERR_TIMEOUT_MMA, 1)) { done_ok = false; break; }
            tc_fence_after();
            {   // S = S Diag(exp(G_C)) + ΔS (fp32 master), tf32 copy back to TMEM
                const float *gcb = m->gcb[par];
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    uint32_t x[32];
                    tmem_ld32(tmem + lane_off + TM_DS + half * 64 + part * 32, x);
                    tmem_wait_ld();
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const float gc = CHANNEL ? gcb[half * 64 + part * 32 + jj] : gcb[0];
                        const float sv = fmaf(gc, S[part * 32 + jj], __uint_as_float(x[jj]));
                        S[part * 32 + jj] = sv;
                        x[jj] = to_tf32(sv);
                    }
                    tmem_st32(tmem + lane_off + TM_S + half * 64 + part * 32, x);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            group_sync(1);
        }
        if (done_ok && nchunks > 0) {
            tc_fence_after();
            store_o(nchunks - 1);
        }
        if (fin != nullptr) {
#pragma unroll
            for (int j = 0; j < 64; j += 4)
                *reinterpret_cast<float4 *>(fin + sg + j) =
                    make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    } else {
        // ====================================================== prep group ====
        const int p = tid - 256;
        bool tma_pending = false;
        uint32_t ph_tma = 0, ph_p = 0;

        // gates and beta run ahead of the tiles: scalar gates two chunks ahead in
        // registers (prep warp 0), channel gates one chunk ahead in registers and
        // two chunks ahead in L2
        float gs0 = 0.f, gs1 = 0.f, bs0 = 0.f, bs1 = 0.f;   // chunk c (prep warp 0)
        float fg0 = 0.f, fg1 = 0.f, fb0 = 0.f, fb1 = 0.f;   // chunk c + 1 (scalar gates)
        float gr[32];                                        // channel gates (KDA)
#pragma unroll
        for (int k = 0; k < 32; ++k) gr[k] = 0.f;
        const int ch = p & 127, hh = p >> 7;                 // KDA: channel, token half
        auto load_scalar = [&](int c, float &ga, float &gb, float &ba, float &bb) {
            if (p < 32 && c < nchunks) {
                const int tok0 = t0 + c * C;
                const int cl = min(C, len - c * C);
                const int i0 = 2 * p, i1 = 2 * p + 1;
                const size_t r0 = (size_t)(tok0 + i0) * H + h, r1 = (size_t)(tok0 + i1) * H + h;
                ba = i0 < cl ? beta[r0] : 0.f;
                bb = i1 < cl ? beta[r1] : 0.f;
                if (!CHANNEL) {   // raw values: clamped where used, so nothing waits here
                    ga = i0 < cl ? g[r0] : 0.f;
                    gb = i1 < cl ? g[r1] : 0.f;
                }
            }
        };
        auto load_channel = [&](int c) {
            if (CHANNEL && c < nchunks) {
                const int tok0 = t0 + c * C;
                const int cl = min(C, len - c * C);
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const int i = hh * 32 + k;
                    gr[k] = i < cl ? g[((size_t)(tok0 + i) * H + h) * D + ch] : 0.f;
                }
            }
        };
        auto l2_channel = [&](int c) {   // one 128-byte line of chunk c's gate rows per thread
            if (CHANNEL && c < nchunks) {
                const int tok0 = t0 + c * C;
                const int i = p >> 2;
                if (i < len - c * C) {
                    const float *a = g + ((size_t)(tok0 + i) * H + h) * D + (p & 3) * 32;
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(a));
                }
            }
        };
        auto issue_tma = [&](int c) {
            const int tok0 = t0 + c * C;
            if (c + 1 < nchunks) {       // warm L2 with the chunk after this one
                const int t1 = tok0 + C;
                tma_prefetch_l2_3d(&tm_k, 0, hq, t1);
                tma_prefetch_l2_3d(&tm_k, 64, hq, t1);
                tma_prefetch_l2_3d(&tm_q, 0, hq, t1);
                tma_prefetch_l2_3d(&tm_q, 64, hq, t1);
                tma_prefetch_l2_3d(&tm_v, 0, h, t1);
                tma_prefetch_l2_3d(&tm_v, 64, h, t1);
            }
            fence_proxy_async();
            mbar_arrive_expect_tx(&m->bar_tma, 6 * 8192);
            tma_load_3d(sm + OFF_KQ + 0, &tm_k, &m->bar_tma, 0, hq, tok0);
            tma_load_3d(sm + OFF_KQ + 16384, &tm_k, &m->bar_tma, 64, hq, tok0);
            tma_load_3d(sm + OFF_KQ + 8192, &tm_q, &m->bar_tma, 0, hq, tok0);
            tma_load_3d(sm + OFF_KQ + 24576, &tm_q, &m->bar_tma, 64, hq, tok0);
            tma_load_3d(sm + OFF_V + 0, &tm_v, &m->bar_tma, 0, h, tok0);
            tma_load_3d(sm + OFF_V + 8192, &tm_v, &m->bar_tma, 64, h, tok0);
        };
        if (nchunks > 0) {
            if (p == 0) {
                issue_tma(0);
                tma_pending = true;
            }
            load_scalar(0, gs0, gs1, bs0, bs1);
            load_scalar(1, fg0, fg1, fb0, fb1);
            l2_channel(0);
            l2_channel(1);
        }

        for (int c = 0; c < nchunks; ++c) {
            const uint32_t par = c & 1;
            float GC = 0.f, R = 0.f;

            // ---- a2: gates ----------------------------------------------------
            if (p < 32) {
                m->u.s.beta[2 * p] = bs0;       // beta is first in both layouts
                m->u.s.beta[2 * p + 1] = bs1;
            }
            if (p == 0) m->slow = 0;
            if (!CHANNEL) {
                if (p < 32) {
                    const int i0 = 2 * p, i1 = 2 * p + 1;
                    gs0 = clamp_log_gate(gs0);
                    gs1 = clamp_log_gate(gs1);
                    const float pair = gs0 + gs1;
                    float incl = pair;
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const float y = __shfl_up_sync(0xffffffffu, incl, off);
                        if (lane >= off) incl += y;
                    }
                    const float G0 = incl - pair + gs0, G1 = incl;
                    const float Gl = __shfl_sync(0xffffffffu, incl, 31);
                    m->u.s.G[i0] = G0; m->u.s.G[i1] = G1;
                    const float e0 = __expf(G0), e1 = __expf(G1);
                    m->u.s.gam[i0] = e0; m->u.s.gam[i1] = e1;
                    m->u.s.kp[i0] = bs0 * e0; m->u.s.kp[i1] = bs1 * e1;
                    m->u.s.kh[i0] = __expf(Gl - G0); m->u.s.kh[i1] = __expf(Gl - G1);
                    m->u.s.ieg[i0] = __expf(-G0); m->u.s.ieg[i1] = __expf(-G1);
                    if (p == 0) m->wide = (Gl < -80.f) ? 1 : 0;
                }
            } else {
                // this chunk's channel gates (L2-resident: prefetched two chunks ago),
                // then the inclusive cumsum of this thread's 32 tokens of channel ch
                load_channel(c);
                gr[0] = clamp_log_gate(gr[0]);
#pragma unroll
                for (int k = 1; k < 32; ++k) gr[k] = clamp_log_gate(gr[k]) + gr[k - 1];
                if (hh == 0) m->u.c.T0[ch] = gr[31];
                else m->u.c.T1[ch] = gr[31];
            }
            // roll the scalar pipeline: chunk c+1 moves up, chunk c+2 is requested
            gs0 = fg0; gs1 = fg1; bs0 = fb0; bs1 = fb1;
            load_scalar(c + 2, fg0, fg1, fb0, fb1);
            if (!group_wait(&m->bar_tma, ph_tma, m, err, ERR_TIMEOUT_TMA, 2)) break;
            ph_tma ^= 1;
            tma_pending = false;

            if (CHANNEL) {
                // chunk-cumulative gate of this thread's tokens; reference R = G_31
                const float T0 = m->u.c.T0[ch], T1 = m->u.c.T1[ch];
                if (hh == 1) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) gr[k] += T0;
                }
                R = T0;
                GC = T0 + T1;
                // fp16 P1 operands: rows [K e^{G-R}; Q e^{G-R}] (X2), K e^{R-G} (TM)
                bool bad = false;
                const uint32_t kcol = (ch >> 6) * 16384, bcol = (ch >> 6) * 8192;
                const uint32_t cch = (ch & 63) >> 3, cel = (ch & 7) * 2;
#pragma unroll 4
                for (int k = 0; k < 32; ++k) {
                    const int i = hh * 32 + k;
                    const uint32_t src = sbase + OFF_KQ + kcol + sw128_offset(i, cch) + cel;
                    const float kv = ld_shared_bf16(src), qv = ld_shared_bf16(src + 8192);
                    const float up = __expf(gr[k] - R), dn = __expf(R - gr[k]);
                    const float a = kv * up, b = qv * up, e = kv * dn;
                    bad |= !(fabsf(a) < kF16Limit) || !(fabsf(b) < kF16Limit) ||
                           !(fabsf(e) < kF16Limit);
                    st_shared_b16(sbase + OFF_X2 + kcol + sw128_offset(i, cch) + cel,
                                  __half_as_ushort(__float2half_rn(a)));
                    st_shared_b16(sbase + OFF_X2 + kcol + sw128_offset(64 + i, cch) + cel,
                                  __half_as_ushort(__float2half_rn(b)));
                    st_shared_b16(sbase + OFF_TM + bcol + sw128_offset(i, cch) + cel,
                                  __half_as_ushort(__float2half_rn(e)));
                }
                if (bad) m->slow = 1;
                fence_proxy_async();
                group_sync(2);
            }
            const bool slow = CHANNEL && m->slow != 0;

            // ---- a3: P1 ---------------------------------------------------------
            if (!slow) {
                if (p == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            if (CHANNEL) {
                                mma_f16_ss(tmem + TM_P1W,
                                           sw128_kmajor_desc(sbase + OFF_X2 + kb * 16384 + kk * 32),
                                           sw128_kmajor_desc(sbase + OFF_TM + kb * 8192 + kk * 32),
                                           IDESC_F16, (kb | kk) != 0);
                            } else {
                                const uint32_t a = sbase + OFF_KQ + kb * 16384 + kk * 32;
                                mma_f16_ss(tmem + TM_P1W, sw128_kmajor_desc(a), sw128_kmajor_desc(a),
                                           IDESC_BF16, (kb | kk) != 0);
                            }
                        }
                    mma_commit(&m->bar_p);
                }
                if (!group_wait(&m->bar_p, ph_p, m, err, ERR_TIMEOUT_MMA, 2)) break;
                ph_p ^= 1;
                tc_fence_after();
            }
            // P slot `par` and U slot `par` were last used by chunk c-2's chain;
            // chunk c-1's S1 completing implies that chain finished.
            if (c >= 1 && !group_wait(&m->bar_s1, (c - 1) & 1, m, err, ERR_TIMEOUT_HANDOFF, 2)) break;

            float *Af;
            float *Tf;
            float *Xs;
            const uint32_t pm = sbase + OFF_PM + par * 16384;
            if (!slow) {
                Af = reinterpret_cast<float *>(sm + OFF_X2);
                Tf = reinterpret_cast<float *>(sm + OFF_X2 + 16384);
                Xs = reinterpret_cast<float *>(sm + OFF_TM);
                uint32_t x[32];
                tmem_ld32(tmem + lane_off + TM_P1W + half * 32, x);
                tmem_wait_ld();
                // decay factor exp(G_i - G_j): a product of per-row and per-column
                // factors when the chunk's total decay stays within e^-80 (the
                // factors are then finite normals), else one exponential each
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
                    if (row < C) {
                        st4(Af, i, j0, make_float4(v4[0], v4[1], v4[2], v4[3]));
                    } else {
                        st_shared_v4(pm + half * 8192 + sw128_offset(i, q), to_tf32(v4[0]),
                                     to_tf32(v4[1]), to_tf32(v4[2]), to_tf32(v4[3]));
                    }
                }
            } else {
                // exact A and P on CUDA cores: G [64][128] fp32 in X2, A in TM
                float *Gs = reinterpret_cast<float *>(sm + OFF_X2);
                Af = reinterpret_cast<float *>(sm + OFF_TM);
                Tf = reinterpret_cast<float *>(sm + OFF_X2);
                Xs = reinterpret_cast<float *>(sm + OFF_X2 + 16384);
#pragma unroll
                for (int k = 0; k < 32; ++k) Gs[(hh * 32 + k) * D + ch] = gr[k];
                group_sync(2);
                for (int pr = p; pr < C * (C + 1) / 2; pr += 256) {
                    int i = (int)((sqrtf(8.f * (float)pr + 1.f) - 1.f) * 0.5f);
                    while (i * (i + 1) / 2 > pr) --i;
                    while ((i + 1) * (i + 2) / 2 <= pr) ++i;
                    const int j = pr - i * (i + 1) / 2;
                    float dk = 0.f, dq = 0.f;
                    for (int cc = 0; cc < D; ++cc) {
                        const uint32_t kc = (cc >> 6) * 16384, chk = (cc & 63) >> 3, el = (cc & 7) * 2;
                        const float ki = ld_shared_bf16(sbase + OFF_KQ + kc + sw128_offset(i, chk) + el);
                        const float qi = ld_shared_bf16(sbase + OFF_KQ + kc + 8192 + sw128_offset(i, chk) + el);
                        const float kj = ld_shared_bf16(sbase + OFF_KQ + kc + sw128_offset(j, chk) + el);
                        const float e = __expf(Gs[i * D + cc] - Gs[j * D + cc]) * kj;
                        dk = fmaf(ki, e, dk);
                        dq = fmaf(qi, e, dq);
                    }
                    Af[ax(i, j)] = (j < i) ? m->u.c.beta[i] * dk : 0.f;
                    st_shared_b32(pm + (j >> 5) * 8192 + sw128_offset(i, (j & 31) >> 2) + (j & 3) * 4,
                                  to_tf32(dq));
                }
                for (int e = p; e < C * C; e += 256) {
                    const int i = e >> 6, j = e & 63;
                    if (j > i) {
                        Af[ax(i, j)] = 0.f;
                        st_shared_b32(pm + (j >> 5) * 8192 + sw128_offset(i, (j & 31) >> 2) + (j & 3) * 4,
                                      0u);
                    }
                }
            }
            group_sync(2);

            // ---- a4: T = (I + A)^-1 -------------------------------------------------
            unit_lower_inverse(Af, Tf, Xs, sbase + OFF_TM, p);
            group_sync(2);

            // ---- a5 operands (X1, QT, KH are free once chunk c-1's S3 is done) --------
            if (c >= 1 && !group_wait(&m->bar_s3, (c - 1) & 1, m, err, ERR_TIMEOUT_HANDOFF, 2)) break;
            if (!CHANNEL) {
                if (p == 0) m->gcb[par][0] = __expf(m->u.s.G[C - 1]);
                const int i = p & 63;
                const float kp = m->u.s.kp[i], bt = m->u.s.beta[i], kh = m->u.s.kh[i],
                            gq = m->u.s.gam[i];
                const uint32_t tcol = (i >> 5) * 16384;
                const uint32_t tchunk = (i & 31) >> 2, tel = (i & 3) * 4;
#pragma unroll 1
                for (int it = 0; it < 4; ++it) {
                    const int jc = (p >> 6) + 4 * it;
                    const uint32_t kb = jc >> 3, chk = jc & 7;
                    float kf[8], qf[8], vf[8];
                    bf16x8_to_f32(ld_shared_v4(sbase + OFF_KQ + kb * 16384 + sw128_offset(i, chk)), kf);
                    bf16x8_to_f32(ld_shared_v4(sbase + OFF_KQ + kb * 16384 + 8192 + sw128_offset(i, chk)), qf);
                    bf16x8_to_f32(ld_shared_v4(sbase + OFF_V + kb * 8192 + sw128_offset(i, chk)), vf);
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
            } else {
                if (hh == 0) m->gcb[par][ch] = __expf(GC);
                const uint32_t kcol = (ch >> 6) * 16384, cch = (ch & 63) >> 3, cel = (ch & 7) * 2;
                const uint32_t vcol = (ch >> 6) * 8192;
                const uint32_t rowblk = hh * 16384;
                const uint32_t qaddr = sbase + OFF_QT + (ch >> 5) * 8192 + (ch & 3) * 4;
                const uint32_t qch = (ch & 31) >> 2;
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                    uint32_t wk[4], wh[4], wv[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int k = q4 * 4 + e, i = hh * 32 + k;
                        const uint32_t src = sbase + OFF_KQ + kcol + sw128_offset(i, cch) + cel;
                        const float kv = ld_shared_bf16(src), qv = ld_shared_bf16(src + 8192);
                        const float vv = ld_shared_bf16(sbase + OFF_V + vcol + sw128_offset(i, cch) + cel);
                        const float bi = m->u.c.beta[i];
                        const float eg = __expf(gr[k]);
                        wk[e] = to_tf32(bi * kv * eg);
                        wh[e] = to_tf32(kv * __expf(GC - gr[k]));
                        wv[e] = to_tf32(bi * vv);
                        st_shared_b32(qaddr + sw128_offset(i, qch), to_tf32(qv * eg));
                    }
                    st_shared_v4(sbase + OFF_X1 + rowblk + sw128_offset(ch, q4), wk[0], wk[1], wk[2], wk[3]);
                    st_shared_v4(sbase + OFF_KH + rowblk + sw128_offset(ch, q4), wh[0], wh[1], wh[2], wh[3]);
                    st_shared_v4(sbase + OFF_X2 + rowblk + sw128_offset(ch, q4), wv[0], wv[1], wv[2], wv[3]);
                }
            }
            fence_proxy_async();
            group_sync(2);

            // ---- a5 (tensor part): W^T, Ũ^T -------------------------------------------
            if (p == 0) {
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t kb = k >> 2, kk = k & 3;
                    const uint64_t bd = sw128_kmajor_desc(sbase + OFF_TM + kb * 8192 + kk * 32);
                    mma_tf32_ss(tmem + TM_P1W, sw128_kmajor_desc(sbase + OFF_X1 + kb * 16384 + kk * 32),
                                bd, IDESC_N64, k != 0);
                    mma_tf32_ss(tmem + TM_U0 + par * 64,
                                sw128_kmajor_desc(sbase + OFF_X2 + kb * 16384 + kk * 32), bd, IDESC_N64,
                                k != 0);
                }
                mma_commit(&m->bar_p);
            }
            // the chunk tiles are consumed: stage the next chunk while P2 runs
            if (c + 1 < nchunks) {
                if (p == 0) {
                    issue_tma(c + 1);
                    tma_pending = true;
                }
                l2_channel(c + 2);
            }
            if (!group_wait(&m->bar_p, ph_p, m, err, ERR_TIMEOUT_MMA, 2)) break;
            ph_p ^= 1;
            tc_fence_after();

            // -W -> [tok][dk] tf32 operand (thread = d_k row of W^T)
            {
                uint32_t x[32];
                tmem_ld32(tmem + lane_off + TM_P1W + half * 32, x);
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
            group_sync(2);
            if (p == 0) mbar_arrive(&m->bar_ready);
        }
        // never leave a TMA load in flight into this CTA's shared memory
        if (p == 0 && tma_pending) (void)mbar_wait(&m->bar_tma, ph_tma);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host ----

}  // namespace

bool tcgen05_prefill_available() { return true; }

bool tcgen05_prefill_serves(bool) { return true; }

size_t tcgen05_workspace_bytes(int, int, int) { return 16; }

cudaError_t launch_prefill_tcgen05(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, const float *h0, const int32_t *cu,
                                   int num_seqs, int total_T, int Hqk, int H, bool channel,
                                   void *o, float *fin, void *workspace, cudaStream_t stream) {
    uint32_t *err = static_cast<uint32_t *>(workspace);
    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(uint32_t), stream);
    if (e != cudaSuccess) return e;
    if ((size_t)num_seqs * H == 0) return cudaSuccess;
    if (total_T == 0) {
        // nothing to stage: the state passes through unchanged
        return launch_prefill_simt(q, k, v, g, beta, h0, cu, num_seqs, total_T, Hqk, H, D, D,
                                   channel, true, o, fin, stream);
    }
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, total_T, Hqk) || !make_map(&mk, k, total_T, Hqk) ||
        !make_map(&mv, v, total_T, H))
        return cudaErrorInvalidValue;
    auto kern = channel ? prefill_tc_kernel<true> : prefill_tc_kernel<false>;
    e = ensure_dynamic_smem(reinterpret_cast<const void *>(kern), (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const size_t blocks = (size_t)num_seqs * H;
    if (blocks > 0x7fffffffull) return cudaErrorInvalidConfiguration;
    kern<<<(unsigned)blocks, kThreads, SMEM_BYTES, stream>>>(
        mq, mk, mv, g, beta, h0, cu, num_seqs, total_T, Hqk, H, static_cast<__nv_bfloat16 *>(o),
        fin, err);
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

// A wait on a flag that nothing sets, bounded by `polls` checks; when it
// gives up it records the failure in the scratch's error word exactly as a
// prefill kernel's bounded wait does.  The flag is a word of the scratch that
// no code writes, so it stays zero.
__global__ void noalloc_wait_probe_kernel(uint32_t polls) {
    volatile uint32_t *flag = reinterpret_cast<volatile uint32_t *>(g_noalloc_scratch + 128);
    uint32_t *err = reinterpret_cast<uint32_t *>(g_noalloc_scratch);
    for (uint32_t it = 0; it < polls; ++it) {
        if (*flag != 0u) return;
        __nanosleep(64);
    }
    atomicOr(err, 1u);
}

}  // namespace
}  // namespace gdr

extern "C" gdr_status_t gdr_prefill_noalloc_check(void *stream) {
    void *scratch = nullptr;
    if (gdr::noalloc_scratch_address(&scratch) != cudaSuccess) return GDR_ERR_CUDA;
    uint32_t word = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(&word, scratch, sizeof(word), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    // the word reports failures since the previous check: clear it
    if (e == cudaSuccess && word != 0) e = cudaMemsetAsync(scratch, 0, sizeof(word), s);
    if (e != cudaSuccess) return GDR_ERR_CUDA;
    return word == 0 ? GDR_OK : GDR_ERR_DEVICE_TIMEOUT;
}

extern "C" gdr_status_t gdr_test_noalloc_wait_timeout(uint32_t polls, void *stream) {
    if (polls == 0 || polls > (1u << 20)) return GDR_ERR_INVALID_ARG;
    void *scratch = nullptr;
    if (gdr::noalloc_scratch_address(&scratch) != cudaSuccess) return GDR_ERR_CUDA;
    gdr::noalloc_wait_probe_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(polls);
    return cudaGetLastError() == cudaSuccess ? GDR_OK : GDR_ERR_CUDA;
}

extern "C" gdr_status_t gdr_prefill_chunked_noalloc(
    const void *q, const void *k, const void *v, const float *g, const float *beta,
    const float *initial_state, const int32_t *cu_seqlens, int32_t num_seqs, int32_t total_T,
    int32_t H, int32_t d_k, int32_t d_v, gdr_gate_mode_t gate_mode, gdr_dtype_t io_dtype, void *o,
    float *final_state, void *stream) {
    // the fixed scratch serves the single-kernel plans only (GDR_ERR_WORKSPACE
    // if this problem needs more)
    gdr_prefill_path_t plan;
    gdr_status_t st = gdr_prefill_plan(num_seqs, total_T, H, d_k, d_v, gate_mode, io_dtype,
                                       gdr::kNoAllocScratchBytes, &plan);
    if (st != GDR_OK) return st;
    void *scratch = nullptr;
    if (gdr::noalloc_scratch_address(&scratch) != cudaSuccess) return GDR_ERR_CUDA;
    return gdr_prefill_chunked(q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, total_T, H,
                               d_k, d_v, gate_mode, io_dtype, o, final_state, scratch,
                               gdr::kNoAllocScratchBytes, stream);
}

