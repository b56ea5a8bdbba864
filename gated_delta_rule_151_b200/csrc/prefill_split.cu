// Chunk-parallel plan of the tensor-core prefill (bf16 I/O, d_k = d_v = 128):
// a prep kernel over every chunk of every head, then a chain kernel that
// carries the state from chunk to chunk with ONE tensor-core product on its
// critical path.
//
// The chunk algebra follows the recurrence on the page "How the New Flash
// Models Work: Inside GLM-5.3-Flash and Qwen3.8-Flash-Next" (section "Linear
// attention: a fixed-size memory in place of the cache", the Gated DeltaNet
// and Kimi Delta Attention equations), rearranged per chunk of C = 64
// tokens.  With S the state entering the chunk, G the within-chunk
// cumulative log-gate and Γ = exp(G):
//
//   A_ij = β_i k_i^T Diag(e^{G_i - G_j}) k_j (j < i),  T = (I + A)^-1
//   W = T diag(β)(K ⊙ Γ),  Ũ = T diag(β) V,  K̂_j = k_j ⊙ e^{G_C - G_j}
//   P_ij = q_i^T Diag(e^{G_i - G_j}) k_j (j <= i),  Q̃_i = q_i ⊙ Γ_i
//
// and the chunk's effect on the state is the affine map
//
//   S' = S Diag(Γ_C) + S N + B,     N = -W^T K̂,  B = Ũ^T K̂
//   O  = S Q'^T + O⁰,               Q' = Q̃ - P W,  O⁰ = P Ũ
//
// (the usual U = Ũ - W S^T, O = Q̃ S^T + P U, S' = S Diag(Γ_C) + U^T K̂,
// with U substituted).  Everything except the products with S depends on
// one chunk only:
//
//   prep kernel   one CTA per (chunk, sequence, head), two CTAs per SM.
//                 TMA stages the bf16 tiles; tcgen05 MMAs form [K;Q] K^T
//                 (A and P), then, after the 64 x 64 inverse on CUDA cores,
//                 W^T and Ũ^T (the bf16 K and V tiles are the MN-major A
//                 operands as TMA left them; T diag(β) is split into a bf16
//                 high and low part), then N^T = K̂^T (-W) and P (-W) with W
//                 split into fp16 high and low parts, then P Ũ.  It writes a
//                 chunk record: N^T, the K̂ tile, Ũ^T, Q' and O⁰ as fp16
//                 images with power-of-two scales, and exp(G_C).
//   chain kernel  one CTA per (sequence, head).  Per chunk: D_B = Ũ^T K̂
//                 (issued early, off the critical path), D_S = S N with S as
//                 fp16 high + low parts in TMEM, D_O = S Q'^T; the state
//                 warps form S' from D_S and D_B in fp32 and write the new
//                 S halves back to TMEM, which starts the next chunk's D_S;
//                 the output warps add O⁰ and store o.
//
// Splitting S, W and T diag(β) into high and low halves keeps the state's
// rounding at about 2^-22 where a single fp16 or tf32 rounding per chunk
// would be amplified by the conditioning of I + A (up to ~10 at beta = 2).
// Records take 98,848 bytes per (chunk, head); problems whose records exceed
// 8 GiB run in windows of chunks, the state passing between windows
// through the workspace.
//
// Because the chunk map is affine, a run of chunks composes into one affine
// map as well.  With few (sequence, head) chains the chain is cut into
// segments: a first launch runs segment 0 from the initial state and every
// middle segment twice, from a zero state (its B_s) and from the identity
// without B (its transition M_s); a small fp32 kernel chains
// S_in(s + 1) = S_in(s) M_s + B_s; a second launch runs every later segment
// in full from its incoming state.  With at most 64 chains and one window,
// the step is instead cut into pieces of chunks whose prep runs beside the
// previous piece's chain on helper streams.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
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
// Byte offsets inside one record.  The operand images are fp16 in the
// 128-byte swizzled layouts the chain kernel's MMA descriptors read (rows of
// 64 halves whose 16-byte chunks are XOR-swizzled by row % 8, blocks
// 1024-byte aligned).  Each image carries its own power-of-two scale 2^s,
// chosen so that its largest magnitude lies in [2^14, 2^15).
constexpr uint32_t REC_NT = 0;        // N^T [j][i]: 2 K-blocks (i 0-63, 64-127) of 128 rows (s_N)
constexpr uint32_t REC_KH = 32768;    // K̂ tile [t][j]: 2 blocks (j 0-63, 64-127) of 64 rows (s_K)
constexpr uint32_t REC_UT = 49152;    // Ũ^T [r][t]: 128 rows (s_U)
constexpr uint32_t REC_QP = 65536;    // Q' [t][j]: 2 K-blocks of 64 rows (s_Q)
constexpr uint32_t REC_OZ = 81920;    // O⁰ [t][r]: plain rows of 256 bytes (s_O)
constexpr uint32_t REC_GC = 98304;    // exp(G_C): 1 float (scalar gate) or 128 (channel gate)
constexpr uint32_t REC_EX = 98816;    // int32 {s_N, s_K, s_U, s_Q, s_O, 0, 0, 0}
constexpr uint32_t REC_BYTES = 98848;
static_assert(REC_BYTES % 16 == 0 && REC_EX + 32 == REC_BYTES, "record layout");

// Byte offset of fp16 element (r, c) (c < 64) inside a block of 128-byte rows.
__host__ __device__ constexpr uint32_t h16_offset(uint32_t r, uint32_t c) {
    return r * 128u + ((((c >> 3) ^ (r & 7u)) & 7u) << 4) + (c & 7u) * 2u;
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

// fp16 high part of two values and the fp16 rounding of what it leaves.
__device__ __forceinline__ void f2h2_hilo(float a, float b, uint32_t &hi, uint32_t &lo) {
    const __half2 h = __floats2half2_rn(a, b);
    const float2 back = __half22float2(h);
    const __half2 l = __floats2half2_rn(a - back.x, b - back.y);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
}

// bf16 high part of two values and the bf16 rounding of what it leaves.
__device__ __forceinline__ void bf2_hilo(float a, float b, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    const float2 back = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(a - back.x, b - back.y);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
}

__device__ __forceinline__ uint16_t bf16_bits(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// Shared-memory accesses through ordinary pointers (byte offsets into the
// CTA's dynamic shared memory), so that the compiler may batch and reorder
// them; every hand-off to the tensor cores or to other threads still goes
// through a fence or barrier that orders memory.
__device__ __forceinline__ float smb16(const uint8_t *sm, uint32_t off) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(sm + off));
}
__device__ __forceinline__ void smh16(uint8_t *sm, uint32_t off, float v) {
    *reinterpret_cast<__half *>(sm + off) = __float2half_rn(v);
}
__device__ __forceinline__ void smu16(uint8_t *sm, uint32_t off, uint16_t v) {
    *reinterpret_cast<uint16_t *>(sm + off) = v;
}
__device__ __forceinline__ uint4 smv4(const uint8_t *sm, uint32_t off) {
    return *reinterpret_cast<const uint4 *>(sm + off);
}
__device__ __forceinline__ void smv4(uint8_t *sm, uint32_t off, uint32_t a, uint32_t b, uint32_t c,
                                     uint32_t d) {
    *reinterpret_cast<uint4 *>(sm + off) = make_uint4(a, b, c, d);
}

// ------------------------------------------------------------- chunk map ----
// Chunks are numbered globally, sequence after sequence: sequence n owns
// global chunks base[n] .. base[n+1] - 1, base computed on the device from
// cu_seqlens (or the equal lengths).  The record of (global chunk, head) sits
// at slot (gc - w0) * H + h of the resident window [w0, w1).  A launch covers
// either a window of global chunks (by_window) or the local chunks c0 .. c1-1
// of every sequence (a pipeline piece, when one window holds every record).
struct ChunkMap {
    const int32_t *base;   // device [num_seqs + 1]
    int w0, w1;            // resident global chunks
    int c0, c1;            // local chunks of every sequence
    int win;               // window index (state slots between windows)
    int by_window;
    // Segmented scan (few chains): every sequence is cut into nseg segments of
    // ceil(chunks / nseg) chunks.  Phase 1 runs segment 0 in full from the
    // initial state and, for segments 1 .. nseg-2, the chain from a zero state
    // (its B) and the transition from the identity without B (its M); phase 2
    // runs segments 1 .. nseg-1 in full from their composed incoming states.
    int nseg;              // 0: no segments
    int phase;             // 1 or 2
    float *slots;          // [chains][nseg][3][D * D]: incoming state, B, M
};

// base[n] = sum over m < n of the chunk count of sequence m (exclusive
// prefix sum, one CTA of 1024 threads); base[num_seqs] = total chunks.
__global__ void __launch_bounds__(1024)
chunk_base_kernel(const int32_t *__restrict__ cu, int num_seqs, int total_T, int32_t *base) {
    __shared__ int wsum[32];
    __shared__ int carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int start = 0; start < num_seqs; start += 1024) {
        const int n = start + tid;
        int v = 0;
        if (n < num_seqs) {
            int t0, len;
            sequence_range(cu, n, num_seqs, total_T, t0, len);
            v = (len + C - 1) / C;
        }
        int x = v;   // inclusive scan within the warp
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, off);
            if (lane >= off) x += y;
        }
        if (lane == 31) wsum[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int w = wsum[lane];
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, off);
                if (lane >= off) w += y;
            }
            wsum[lane] = w;   // inclusive over warps
        }
        __syncthreads();
        const int before = carry + (warp > 0 ? wsum[warp - 1] : 0);
        if (n < num_seqs) base[n] = before + x - v;
        __syncthreads();
        if (tid == 0) carry += wsum[31];
        __syncthreads();
    }
    if (tid == 0) base[num_seqs] = carry;
}

// Segment composition: S_in(s + 1) = S_in(s) M_s + B_s for s = 1 .. nseg-2,
// in fp32.  The rows of a state are independent, so CTA (chain, rb) owns rows
// 16 rb .. 16 rb + 15 for the whole recurrence and keeps them in shared
// memory, transposed (st[k][16]), from one step to the next; thread tid holds
// rows 4 (tid / 32) .. +3 by columns 4 (tid % 32) .. +3 in registers.  M_s is
// staged in shared memory with 16-byte asynchronous copies, the next step's
// while this step multiplies.
constexpr int kComposeThreads = 128;
constexpr uint32_t COMPOSE_SMEM = (2 * D * D + 16 * D) * sizeof(float);   // 136 KiB
__device__ __forceinline__ void async_copy16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__global__ void __launch_bounds__(kComposeThreads)
segment_compose_kernel(float *__restrict__ slots, int nseg) {
    extern __shared__ __align__(16) float csm[];
    float *st = csm + 2 * D * D;
    const int chain = blockIdx.x, rb = blockIdx.y, tid = threadIdx.x;
    const int r0 = (tid >> 5) * 4, c0 = (tid & 31) * 4;
    auto slot = [&](int sg, int kind) {
        return slots + (((size_t)chain * nseg + sg) * 3 + kind) * D * D;
    };
    auto stage_m = [&](int sg) {
        const float *M = slot(sg, 2);
        float *dst = csm + (sg & 1) * D * D;
#pragma unroll 8
        for (int e = tid; e < D * D / 4; e += kComposeThreads) async_copy16(dst + 4 * e, M + 4 * e);
        async_commit();
    };
    stage_m(1);
    {   // incoming rows of segment 1 (segment 0's final state), transposed
        const float *Sin = slot(1, 0) + (size_t)rb * 16 * D;
        float4 x[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            x[i] = *reinterpret_cast<const float4 *>(Sin + (size_t)(r0 + i) * D + c0);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            st[(c0 + 0) * 16 + r0 + i] = x[i].x; st[(c0 + 1) * 16 + r0 + i] = x[i].y;
            st[(c0 + 2) * 16 + r0 + i] = x[i].z; st[(c0 + 3) * 16 + r0 + i] = x[i].w;
        }
    }
    for (int sg = 1; sg + 1 < nseg; ++sg) {
        const float *B = slot(sg, 1) + (size_t)rb * 16 * D;
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 b = *reinterpret_cast<const float4 *>(B + (size_t)(r0 + i) * D + c0);
            acc[i][0] = b.x; acc[i][1] = b.y; acc[i][2] = b.z; acc[i][3] = b.w;
        }
        if (sg + 2 < nseg) { stage_m(sg + 1); async_wait<1>(); }
        else async_wait<0>();
        __syncthreads();   // M_sg and the incoming rows are in shared memory
        const float *Ms = csm + (sg & 1) * D * D;
#pragma unroll 8
        for (int k = 0; k < D; ++k) {
            const float4 a = *reinterpret_cast<const float4 *>(st + k * 16 + r0);
            const float4 m = *reinterpret_cast<const float4 *>(Ms + k * D + c0);
            const float av[4] = {a.x, a.y, a.z, a.w}, mv[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], mv[j], acc[i][j]);
        }
        __syncthreads();   // every thread is done with st and M_sg
        float *Sout = slot(sg + 1, 0) + (size_t)rb * 16 * D;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            *reinterpret_cast<float4 *>(Sout + (size_t)(r0 + i) * D + c0) =
                make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
#pragma unroll
            for (int j = 0; j < 4; ++j) st[(c0 + j) * 16 + r0 + i] = acc[i][j];
        }
    }
}

// ------------------------------------------------------------ prep kernel ----
constexpr int kPrepThreads = 256;
// Shared memory (two CTAs per SM).  Regions and what they hold in turn:
constexpr uint32_t PO_KQ = 0;       // bf16 [K d0-63][Q d0-63][K d64-127][Q d64-127] (TMA);
                                    //   channel gate: K' = K ⊙ Γ (bf16 high) over K, Q̃ fp16 over Q
constexpr uint32_t PO_V = 32768;    // bf16 [V d0-63][V d64-127] (TMA); after P2: Ũ^T fp16
constexpr uint32_t PO_RA = 49152;   // A fp32 / channel P1 A operand (with RT) / slow-path G (with RT);
                                    //   then T diag(.) bf16 high | low; after P2: -W^T fp16 high
constexpr uint32_t PO_RT = 65536;   // T fp32; then the K̂ fp16 tile
constexpr uint32_t PO_RX = 81920;   // inverse scratch / channel P1 B operand / slow-path A; then
                                    //   scalar T diag(β) bf16 high | low, channel K' bf16 low;
                                    //   after P2: -W^T fp16 low
constexpr uint32_t PO_P = 98304;    // P fp16 [i][j] (rows 64-127 of the M = 128 A operand whose
                                    //   rows 0-63 are the 8 KiB before it, never read back)
constexpr uint32_t PO_MISC = 106496;
constexpr uint32_t PREP_SMEM = PO_MISC + 2560;   // 109056: two CTAs per SM
constexpr uint32_t PT_W = 0, PREP_TMEM_COLS = 256;   // P1 accumulates at column 0
constexpr uint32_t IDESC_P2 = make_idesc(1, 128, 64) | kIdescAMN;     // bf16, A MN-major
constexpr uint32_t IDESC_NT = make_idesc(0, 128, 128) | kIdescAMN;    // fp16, A MN-major
constexpr uint32_t IDESC_H128 = make_idesc(0, 128, 128);              // fp16, K-major
constexpr uint32_t IDESC_H64 = make_idesc(0, 128, 64);

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
            float beta[C], T[4][D];    // chunk gate totals of each 16-token quarter
        } c;
    } u;                               // beta comes first in both layouts
    float red[3][8];                   // per-warp maxima for the image scales
};
static_assert(sizeof(PrepMisc) <= 2560, "prep misc area overflow");
static_assert(offsetof(PrepMisc, u) % 16 == 0, "prep misc arrays misaligned");

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

// Block-wide maxima of three per-thread values (all >= 0); all 256 threads
// call it (two __syncthreads inside) and receive the same three results.
__device__ __forceinline__ void block_max3(float (&v)[3], float (*red)[8]) {
    const int w = threadIdx.x >> 5;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        const uint32_t u = __reduce_max_sync(0xffffffffu, __float_as_uint(v[k]));
        if ((threadIdx.x & 31) == 0) red[k][w] = __uint_as_float(u);
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        float mx = 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) mx = fmaxf(mx, red[k][q]);
        v[k] = mx;
    }
    __syncthreads();
}

// 2^e for any integer e, saturated to the float range's normal powers.
__device__ __forceinline__ float exp2c(int e) { return exp2i(min(max(e, -126), 126)); }

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

// Fused input-side prologue: the chunk's q, k (query/key head hq) and v
// (value head h) tiles computed from the raw projections instead of loaded.
// Each token is the depthwise causal convolution of kernel size four (page
// "Qwen3.8-Flash-Next and GLM-5.3-Flash share a 3:1 long-context pattern",
// section "Kimi Delta Attention extends recurrent memory control") of the
// token and the three before it, with the incoming convolution state before
// the sequence's first token; then the optional SiLU and the q/k L2 norms
// over the head's 128 channels.
//
// The raw rows of the chunk and the three before it (those inside the
// sequence) are staged in the scratch regions with 16-byte asynchronous
// copies, all in flight together, issued before the CTA sets up its barriers
// and TMEM.  Then warp w computes tokens 8w .. 8w + 7, lane l channels
// 4l .. 4l + 3, with the standalone prologue kernel's arithmetic (packed
// fp32x2 convolution and SiLU, the eight tokens' norms reduced together:
// the same bits), and writes bf16 into the 128-byte-swizzled tile layout the
// TMA loads produce.  Rows past the sequence's end are zero.
constexpr int kStageRows = C + 3;                      // rows c C - 3 .. c C + 63
constexpr uint32_t PO_STAGE = PO_RA;                   // [k, q, v][kStageRows][128] bf16
static_assert(PO_STAGE + 3 * kStageRows * 256 <= PO_MISC, "fused prologue staging overflow");

__device__ __forceinline__ void fused_prologue_stage(const PrologueIn &P, uint8_t *sm, int t0,
                                                     int len, int c, int hq, int h, int Hqk,
                                                     int H) {
#pragma unroll 1
    for (int which = 0; which < 3; ++which) {   // k, q, v
        const __nv_bfloat16 *x =
            static_cast<const __nv_bfloat16 *>(which == 0 ? P.xk : which == 1 ? P.xq : P.xv);
        const int width = which == 2 ? H * D : Hqk * D;
        const __nv_bfloat16 *src = x + (which == 2 ? h : hq) * D;
        uint8_t *dst = sm + PO_STAGE + (uint32_t)which * kStageRows * 256u;
        for (int e = threadIdx.x; e < kStageRows * 16; e += kPrepThreads) {   // 16-byte pieces
            const int r = e >> 4, piece = e & 15;
            const int tau = c * C - 3 + r;
            if (tau >= 0 && tau < len)
                async_copy16(dst + r * 256 + piece * 16, src + (size_t)(t0 + tau) * width + piece * 8);
        }
    }
    async_commit();
}

__device__ __forceinline__ void fused_prologue_tiles(const PrologueIn &P, uint8_t *sm, int n,
                                                     int len, int c, int hq, int h) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cl = min(C, len - c * C);
    async_wait<0>();
    __syncthreads();   // every thread's staged rows have landed

    const int i0 = warp * 8;
    const uint32_t lane_ch = (uint32_t)(lane & 15) >> 1, lane_b = (uint32_t)(lane & 1) * 8u;
#pragma unroll 1
    for (int which = 0; which < 3; ++which) {   // k, q, v
        const bool isv = which == 2;
        const int col = (isv ? h : hq) * D + 4 * lane;            // this lane's first channel
        const float *w = which == 0 ? P.wk : which == 1 ? P.wq : P.wv;
        const int choff = which == 0 ? P.Cq : which == 1 ? 0 : 2 * P.Cq;
        float2 tp[2][4];                                          // [channel pair][tap]
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const float4 a = *reinterpret_cast<const float4 *>(w + (size_t)(col + 2 * j) * 4);
            const float4 b = *reinterpret_cast<const float4 *>(w + (size_t)(col + 2 * j + 1) * 4);
            tp[j][0] = make_float2(a.x, b.x); tp[j][1] = make_float2(a.y, b.y);
            tp[j][2] = make_float2(a.z, b.z); tp[j][3] = make_float2(a.w, b.w);
        }
        // window rows: tokens i0 - 3 .. i0 + 7 of the chunk (sequence positions
        // tau = c C + i); before the sequence the incoming state, past its end 0
        const uint8_t *rows = sm + PO_STAGE + (uint32_t)(which * kStageRows + i0) * 256u + lane * 8;
        float2 xp[11][2];
#pragma unroll
        for (int r = 0; r < 11; ++r) {
            const int tau = c * C + i0 - 3 + r;
            if (tau >= 0 && tau < len) {
                const uint2 raw = *reinterpret_cast<const uint2 *>(rows + r * 256);
                xp[r][0] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
                xp[r][1] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
            } else {
                float v4[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    v4[j] = (tau < 0 && P.state_in != nullptr)
                                ? P.state_in[((size_t)n * P.Call + choff + col + j) * 3 + (tau + 3)]
                                : 0.f;
                xp[r][0] = make_float2(v4[0], v4[1]);
                xp[r][1] = make_float2(v4[2], v4[3]);
            }
        }
        float ss[8];
#pragma unroll
        for (int s = 0; s < 8; ++s) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                float2 acc = __fmul2_rn(tp[j][0], xp[s][j]);
                acc = __ffma2_rn(tp[j][1], xp[s + 1][j], acc);
                acc = __ffma2_rn(tp[j][2], xp[s + 2][j], acc);
                acc = __ffma2_rn(tp[j][3], xp[s + 3][j], acc);
                xp[s][j] = P.silu ? silu2(acc) : acc;   // row s is not read again
            }
            const float2 q2 = __ffma2_rn(xp[s][1], xp[s][1], __fmul2_rn(xp[s][0], xp[s][0]));
            ss[s] = q2.x + q2.y;
        }
        if (P.norm != 0 && !isv) {
            float tot[8];
            norm_sums8(ss, lane, tot);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const float rn = rsqrt_approx(tot[s] + kNormEps);
                xp[s][0] = __fmul2_rn(xp[s][0], make_float2(rn, rn));
                xp[s][1] = __fmul2_rn(xp[s][1], make_float2(rn, rn));
            }
        }
        uint8_t *tile = sm + (which == 0 ? PO_KQ : which == 1 ? PO_KQ + 8192 : PO_V);
        const uint32_t blk = (uint32_t)(lane >> 4) * (isv ? 8192u : 16384u);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            const int i = i0 + s;
            const float2 z = make_float2(0.f, 0.f);
            const bool live = i < cl;
            const __nv_bfloat162 lo = __float22bfloat162_rn(live ? xp[s][0] : z);
            const __nv_bfloat162 hi = __float22bfloat162_rn(live ? xp[s][1] : z);
            uint2 st;
            st.x = *reinterpret_cast<const uint32_t *>(&lo);
            st.y = *reinterpret_cast<const uint32_t *>(&hi);
            *reinterpret_cast<uint2 *>(tile + blk + sw128_offset(i, lane_ch) + lane_b) = st;
        }
    }
}

// A bf16 pair (low half first) as two floats.
__device__ __forceinline__ float2 bf2_to_f2(uint32_t v) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v));
}

// Clamped log-gates of 16 consecutive tokens of two channels -> their running
// sums; the sums' last values (the quarter's totals) go to tot[0..1].
__device__ __forceinline__ void gate_scan16(float2 (&gr)[16], float *tot) {
    gr[0] = make_float2(clamp_log_gate(gr[0].x), clamp_log_gate(gr[0].y));
#pragma unroll
    for (int k = 1; k < 16; ++k)
        gr[k] = make_float2(clamp_log_gate(gr[k].x) + gr[k - 1].x, clamp_log_gate(gr[k].y) + gr[k - 1].y);
    *reinterpret_cast<float2 *>(tot) = gr[15];
}

template <bool CHANNEL, bool FUSED>
__global__ void __launch_bounds__(kPrepThreads, 2)
prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
            const float *__restrict__ g,
            const float *__restrict__ beta, const int32_t *__restrict__ cu, int num_seqs,
            int total_T, int Hqk, int H, const ChunkMap map, uint8_t *__restrict__ recs,
            const PrologueIn pin, uint32_t *err) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = smem_u32(smem_raw);
    int n, h, c, gc;
    if (map.by_window) {
        gc = map.w0 + static_cast<int>(blockIdx.x);
        h = blockIdx.y;
        if (gc >= map.w1 || gc >= map.base[num_seqs]) return;
        int lo = 0, hi = num_seqs;   // base[lo] <= gc < base[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (map.base[mid] <= gc) lo = mid;
            else hi = mid;
        }
        n = lo;
        c = gc - map.base[n];
    } else {
        h = blockIdx.y % H;
        n = blockIdx.y / H;
        c = map.c0 + static_cast<int>(blockIdx.x);
        if (c >= map.base[n + 1] - map.base[n]) return;   // past this sequence's last chunk
        gc = map.base[n] + c;
    }
    const int hq = h / (H / Hqk);
    int t0, len;
    sequence_range(cu, n, num_seqs, total_T, t0, len);
    if (c * C >= len) return;
    if ((sbase & 1023u) != 0) {
        if (threadIdx.x == 0) atomicOr(err, ERR_SMEM_ALIGN);
        return;
    }
    uint8_t *sm = smem_raw;
    PrepMisc *m = reinterpret_cast<PrepMisc *>(sm + PO_MISC);
    uint8_t *rec = recs + ((size_t)(gc - map.w0) * H + h) * REC_BYTES;
    const int tok0 = t0 + c * C;
    const int cl = min(C, len - c * C);

    if (FUSED) fused_prologue_stage(pin, sm, t0, len, c, hq, h, Hqk, H);

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
    // channel gate: the chunk's gates [64 tokens][128 channels] fp32 land in
    // RT and RX (free until the P1 operand pass) with the tiles
    constexpr bool kGateTma = CHANNEL && !FUSED;
    if (!FUSED && tid == 0) {
        mbar_arrive_expect_tx(&m->bar_tma, 6 * 8192 + (kGateTma ? 32768 : 0));
        if (kGateTma) {
#pragma unroll
            for (int j = 0; j < 4; ++j) tma_load_3d(sm + PO_RT + j * 8192, &tm_g, &m->bar_tma, 32 * j, h, tok0);
        }
        tma_load_3d(sm + PO_KQ + 0, &tm_k, &m->bar_tma, 0, hq, tok0);
        tma_load_3d(sm + PO_KQ + 16384, &tm_k, &m->bar_tma, 64, hq, tok0);
        tma_load_3d(sm + PO_KQ + 8192, &tm_q, &m->bar_tma, 0, hq, tok0);
        tma_load_3d(sm + PO_KQ + 24576, &tm_q, &m->bar_tma, 64, hq, tok0);
        tma_load_3d(sm + PO_V + 0, &tm_v, &m->bar_tma, 0, h, tok0);
        tma_load_3d(sm + PO_V + 8192, &tm_v, &m->bar_tma, 64, h, tok0);
    }

    // ---- gates (overlap the tile loads); rows past the sequence end get
    //      beta = 0 and g = 0 ------------------------------------------------
    // channel gate: this thread's channel pair 2 cp, 2 cp + 1 and token quarter
    // qq (tokens 16 qq .. 16 qq + 15); gr = their chunk-cumulative gates
    const int cp = tid & 63, qq = tid >> 6, c0 = 2 * cp;
    float2 gr[16];
    if (!CHANNEL) {
        if (tid < 32) {
            const int i0 = 2 * tid, i1 = 2 * tid + 1;
            const size_t r0 = (size_t)(tok0 + i0) * H + h, r1 = (size_t)(tok0 + i1) * H + h;
            float b0 = 0.f, b1 = 0.f, g0 = 0.f, g1 = 0.f;
            if (FUSED) {
                const float cg = pin.gscale[h];
                if (i0 < cl) { b0 = beta_of(pin.xb[r0]); g0 = clamp_log_gate(log_gate_of(cg, pin.xg[r0])); }
                if (i1 < cl) { b1 = beta_of(pin.xb[r1]); g1 = clamp_log_gate(log_gate_of(cg, pin.xg[r1])); }
            } else {
                if (i0 < cl) { b0 = beta[r0]; g0 = clamp_log_gate(g[r0]); }
                if (i1 < cl) { b1 = beta[r1]; g1 = clamp_log_gate(g[r1]); }
            }
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
        if (FUSED) {
            const float cg = pin.gscale[h];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const int i = qq * 16 + k;
                float2 x = make_float2(0.f, 0.f);
                if (i < cl) {
                    x = *reinterpret_cast<const float2 *>(pin.xg + ((size_t)(tok0 + i) * H + h) * D + c0);
                    x = make_float2(log_gate_of(cg, x.x), log_gate_of(cg, x.y));
                }
                gr[k] = x;
            }
            gate_scan16(gr, m->u.c.T[qq] + c0);
        }
        if (tid < C) {
            const size_t bi = (size_t)(tok0 + tid) * H + h;
            m->u.c.beta[tid] = tid < cl ? (FUSED ? beta_of(pin.xb[bi]) : beta[bi]) : 0.f;
        }
    }

    do {
        if (FUSED) {
            // the tiles from the staged raw rows (their copies overlapped the
            // set-up and the gate loads above)
            fused_prologue_tiles(pin, sm, n, len, c, hq, h);
            fence_proxy_async();   // the tiles are MMA operands
            __syncthreads();
        } else if (!block_wait(&m->bar_tma, 0, &m->abort_flag, err, ERR_TIMEOUT_TMA)) {
            break;
        }

        float kmax = 0.f, qmax = 0.f;   // channel gate: this thread's largest |k| and |q|
        if (kGateTma) {
            // this thread's 2 x 16 gates from the staged rows (row = token, 128
            // bytes per 32 channels), masked past the sequence's end
            const float *gs = reinterpret_cast<const float *>(sm + PO_RT + (cp >> 4) * 8192) + (c0 & 31);
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const int i = qq * 16 + k;
                gr[k] = i < cl ? *reinterpret_cast<const float2 *>(gs + i * 32) : make_float2(0.f, 0.f);
            }
            gate_scan16(gr, m->u.c.T[qq] + c0);
            __syncthreads();   // every quarter's total; the staged gates are read
        }
        float2 GC2 = make_float2(0.f, 0.f);
        if (CHANNEL) {
            // chunk-cumulative gates: the quarters before this one, then the
            // thread's own; reference R = G at token 31 (the end of quarter 1)
            float2 pre = make_float2(0.f, 0.f), R = make_float2(0.f, 0.f);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 t = *reinterpret_cast<const float2 *>(m->u.c.T[q] + c0);
                if (q < qq) pre = make_float2(pre.x + t.x, pre.y + t.y);
                if (q < 2) R = make_float2(R.x + t.x, R.y + t.y);
                GC2 = make_float2(GC2.x + t.x, GC2.y + t.y);
            }
#pragma unroll
            for (int k = 0; k < 16; ++k) gr[k] = make_float2(gr[k].x + pre.x, gr[k].y + pre.y);
            if (qq == 0)
                *reinterpret_cast<float2 *>(rec + REC_GC + c0 * 4) = make_float2(__expf(GC2.x), __expf(GC2.y));
            // fp16 P1 operands: rows [K e^{G-R}; Q e^{G-R}] (RA..RT), K e^{R-G} (RX)
            bool bad = false;
            const uint32_t kcol = (cp >> 5) * 16384, bcol = (cp >> 5) * 8192;
            const uint32_t cch = (cp & 31) >> 2, cel = (cp & 3) * 4;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const int i = qq * 16 + k;
                const uint32_t so = sw128_offset(i, cch) + cel;
                const float2 kv = bf2_to_f2(*reinterpret_cast<const uint32_t *>(sm + PO_KQ + kcol + so));
                const float2 qv = bf2_to_f2(*reinterpret_cast<const uint32_t *>(sm + PO_KQ + kcol + 8192 + so));
                kmax = fmaxf(kmax, fmaxf(fabsf(kv.x), fabsf(kv.y)));
                qmax = fmaxf(qmax, fmaxf(fabsf(qv.x), fabsf(qv.y)));
                const float2 up = make_float2(__expf(gr[k].x - R.x), __expf(gr[k].y - R.y));
                const float2 dn = make_float2(__expf(R.x - gr[k].x), __expf(R.y - gr[k].y));
                const float2 a = __fmul2_rn(kv, up), b = __fmul2_rn(qv, up), e = __fmul2_rn(kv, dn);
                // every value checked on its own: a NaN fails the comparison
                bad |= !(fabsf(a.x) < kF16Limit) || !(fabsf(a.y) < kF16Limit) ||
                       !(fabsf(b.x) < kF16Limit) || !(fabsf(b.y) < kF16Limit) ||
                       !(fabsf(e.x) < kF16Limit) || !(fabsf(e.y) < kF16Limit);
                *reinterpret_cast<uint32_t *>(sm + PO_RA + kcol + so) = f2h2_bits(a.x, a.y);
                *reinterpret_cast<uint32_t *>(sm + PO_RA + kcol + sw128_offset(64 + i, cch) + cel) =
                    f2h2_bits(b.x, b.y);
                *reinterpret_cast<uint32_t *>(sm + PO_RX + bcol + so) = f2h2_bits(e.x, e.y);
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
                                       sw128_kmajor_desc(sbase + PO_RA + kb * 16384 + kk * 32),
                                       sw128_kmajor_desc(sbase + PO_RX + kb * 8192 + kk * 32),
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
        float kbound = 0.f, qbound = 0.f;      // bounds of |K̂| and |Q̃| over the chunk
        // channel gate: this thread's bounds, |K̂| <= max|k| e^{max(G_C - G)} and
        // |Q̃| <= max|q| e^{max G} over its tokens (a bound above the true
        // maximum only moves values down within fp16's normal range)
        float kbnd = 0.f, qbnd = 0.f;
        if (CHANNEL) {
            float dk = -3.0e38f, dq = -3.0e38f;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                dk = fmaxf(dk, fmaxf(GC2.x - gr[k].x, GC2.y - gr[k].y));
                dq = fmaxf(dq, fmaxf(gr[k].x, gr[k].y));
            }
            kbnd = kmax * __expf(dk);
            qbnd = qmax * __expf(dq);
        }
        float *Af;
        float *Tf;
        float *Xs;
        if (!slow) {
            Af = reinterpret_cast<float *>(sm + PO_RA);
            Tf = reinterpret_cast<float *>(sm + PO_RT);
            Xs = reinterpret_cast<float *>(sm + PO_RX);
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
            float mx3[3] = {0.f, 0.f, 0.f};   // |P|; bounds of |K̂| and |Q̃| (see below)
            if (row >= C) {
#pragma unroll
                for (int e = 0; e < 32; ++e) mx3[0] = fmaxf(mx3[0], fabsf(pv[e]));
            }
            if (!CHANNEL) {
                // |K̂| <= max |k| <= max ||k_i||, the diagonal of K K^T; |Q̃| <= max |q|
                if (row < C) {
                    const float kh = m->u.s.kh[i];
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (half * 32 + e == i) mx3[1] = __uint_as_float(x[e]) * kh * kh;
                } else {
                    const float gq = m->u.s.gam[i];
#pragma unroll
                    for (int c8 = 0; c8 < 8; ++c8) {
                        float qf[8];
                        bf16x8_to_f32(smv4(sm, PO_KQ + 8192 + half * 16384 + sw128_offset(i, c8)), qf);
#pragma unroll
                        for (int e = 0; e < 8; ++e) mx3[2] = fmaxf(mx3[2], fabsf(qf[e]) * gq);
                    }
                }
            } else {
                mx3[1] = kbnd;
                mx3[2] = qbnd;
            }
            block_max3(mx3, m->red);
            sP = scale_exp(mx3[0]);
            kbound = CHANNEL ? mx3[1] : sqrtf(mx3[1]);
            qbound = mx3[2];
            if (row >= C) {
                const float f = exp2i(sP);
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const float *v = pv + c4 * 8;
                    st_shared_v4(sbase + PO_P + i * 128 + ((((half * 4 + c4) ^ (i & 7)) & 7) << 4),
                                 f2h2_bits(v[0] * f, v[1] * f), f2h2_bits(v[2] * f, v[3] * f),
                                 f2h2_bits(v[4] * f, v[5] * f), f2h2_bits(v[6] * f, v[7] * f));
                }
            }
        } else {
            // exact A and P on CUDA cores: G [64][128] fp32 in RA..RT, A in RX
            float *Gs = reinterpret_cast<float *>(sm + PO_RA);
            Af = reinterpret_cast<float *>(sm + PO_RX);
            Tf = reinterpret_cast<float *>(sm + PO_RT);
            Xs = reinterpret_cast<float *>(sm + PO_RA);
#pragma unroll
            for (int k = 0; k < 16; ++k) *reinterpret_cast<float2 *>(Gs + (qq * 16 + k) * D + c0) = gr[k];
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
                    st_shared_b16(sbase + PO_P + h16_offset(i, j), 0);
                }
            }
            float mx3[3] = {pm, kbnd, qbnd};
            block_max3(mx3, m->red);
            sP = scale_exp(mx3[0]);
            kbound = mx3[1];
            qbound = mx3[2];
            const float f = exp2i(sP);
#pragma unroll
            for (int it = 0; it < kPairIters; ++it) {
                const int pr = tid + it * kPrepThreads;
                if (pr < C * (C + 1) / 2) {
                    int i, j;
                    pair_ij(pr, i, j);
                    st_shared_b16(sbase + PO_P + h16_offset(i, j), f2h_bits(dqs[it] * f));
                }
            }
        }
        __syncthreads();

        // ---- T = (I + A)^-1 in fp32 (into RT on both paths) ---------------------
        unit_lower_inverse_f32(Af, Tf, Xs, tid);

        // ---- B operands of P2: T diag(f) as bf16 high and low parts, rows t.
        //      Scalar gate: f = β Γ for W (RA) and f = β for Ũ (RX); channel
        //      gate: f = β for both (RA), Γ goes into the A operand ------------
        {
            const float *Tm = reinterpret_cast<const float *>(sm + PO_RT);
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const int item = tid + it * kPrepThreads;
                const int t = item >> 3, cq = item & 7;   // row t, columns 8 cq .. 8 cq + 7
                const float4 a = ld4(Tm, t, cq * 8), b = ld4(Tm, t, cq * 8 + 4);
                const float tv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
                uint32_t h1[4], l1[4], h2[4], l2[4];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const int j = cq * 8 + e;
                    const float x0 = j <= t ? tv[e] : 0.f, x1 = j + 1 <= t ? tv[e + 1] : 0.f;
                    const float b0 = m->u.c.beta[j], b1 = m->u.c.beta[j + 1];
                    if (CHANNEL) {
                        bf2_hilo(x0 * b0, x1 * b1, h1[e / 2], l1[e / 2]);
                    } else {
                        bf2_hilo(x0 * m->u.s.kp[j], x1 * m->u.s.kp[j + 1], h1[e / 2], l1[e / 2]);
                        bf2_hilo(x0 * b0, x1 * b1, h2[e / 2], l2[e / 2]);
                    }
                }
                const uint32_t off = t * 128 + (((cq ^ (t & 7)) & 7) << 4);
                smv4(sm, PO_RA + off, h1[0], h1[1], h1[2], h1[3]);
                smv4(sm, PO_RA + 8192 + off, l1[0], l1[1], l1[2], l1[3]);
                if (!CHANNEL) {
                    smv4(sm, PO_RX + off, h2[0], h2[1], h2[2], h2[3]);
                    smv4(sm, PO_RX + 8192 + off, l2[0], l2[1], l2[2], l2[3]);
                }
            }
        }
        __syncthreads();   // T (RT) is consumed

        // ---- the K̂ tile (fp16, scale s_K) into RT.  Channel gate: also
        //      K' = K ⊙ Γ as bf16 high (over K) and low (RX) parts, and
        //      Q̃ = Q ⊙ Γ as fp16 (scale s_Q) over Q ------------------------------
        sK = scale_exp(kbound);
        if (CHANNEL) sQ = scale_exp(qbound);
        if (!CHANNEL) {
            const float fs = exp2i(sK);
#pragma unroll
            for (int it = 0; it < 4; ++it) {
                const int item = tid + it * kPrepThreads;
                const int blk = item >> 9, t = (item >> 3) & 63, cq = item & 7;
                float kf[8];
                bf16x8_to_f32(smv4(sm, PO_KQ + blk * 16384 + sw128_offset(t, cq)), kf);
                const float f = m->u.s.kh[t] * fs;
                smv4(sm, PO_RT + blk * 8192 + sw128_offset(t, cq),
                             f2h2_bits(kf[0] * f, kf[1] * f), f2h2_bits(kf[2] * f, kf[3] * f),
                             f2h2_bits(kf[4] * f, kf[5] * f), f2h2_bits(kf[6] * f, kf[7] * f));
            }
        } else {
            const float fk = exp2i(sK), fq = exp2i(sQ);
            const uint32_t kcol = (cp >> 5) * 16384, tcol = (cp >> 5) * 8192;
            const uint32_t cch = (cp & 31) >> 2, cel = (cp & 3) * 4;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const int i = qq * 16 + k;
                const uint32_t so = sw128_offset(i, cch) + cel;
                const uint32_t src = PO_KQ + kcol + so, dst = tcol + so;
                const float2 kv = bf2_to_f2(*reinterpret_cast<const uint32_t *>(sm + src));
                const float2 qv = bf2_to_f2(*reinterpret_cast<const uint32_t *>(sm + src + 8192));
                const float2 eg = make_float2(__expf(gr[k].x), __expf(gr[k].y));
                const float2 kh = make_float2(__expf(GC2.x - gr[k].x) * fk, __expf(GC2.y - gr[k].y) * fk);
                const float2 khat = __fmul2_rn(kv, kh);
                *reinterpret_cast<uint32_t *>(sm + PO_RT + dst) = f2h2_bits(khat.x, khat.y);
                const float2 kp = __fmul2_rn(kv, eg);
                uint32_t khi, klo;
                bf2_hilo(kp.x, kp.y, khi, klo);
                *reinterpret_cast<uint32_t *>(sm + src) = khi;
                *reinterpret_cast<uint32_t *>(sm + PO_RX + dst) = klo;
                const float2 qt = __fmul2_rn(__fmul2_rn(qv, eg), make_float2(fq, fq));
                *reinterpret_cast<uint32_t *>(sm + src + 8192) = f2h2_bits(qt.x, qt.y);
            }
        }
        fence_proxy_async();
        __syncthreads();

        // ---- P2: W^T = K'^T (T diag(.))^T and Ũ^T = V^T (T diag(β))^T in bf16,
        //      the K and V tiles (or K' high and low) as MN-major A operands ----
        uint32_t mph = slow ? 0u : 1u;   // next phase of bar_mma
        if (tid == 0) {
            tc_fence_after();
            const uint32_t tb_w = sbase + PO_RA, tb_u = sbase + (CHANNEL ? PO_RA : PO_RX);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t ak = sw128_mnmajor_desc(sbase + PO_KQ + k * 2048, 16384, 1024);
                mma_f16_ss(tmem + 0, ak, sw128_kmajor_desc(tb_w + k * 32), IDESC_P2, k != 0);
                mma_f16_ss(tmem + 0, ak, sw128_kmajor_desc(tb_w + 8192 + k * 32), IDESC_P2, 1);
                if (CHANNEL)
                    mma_f16_ss(tmem + 0, sw128_mnmajor_desc(sbase + PO_RX + k * 2048, 8192, 1024),
                               sw128_kmajor_desc(tb_w + k * 32), IDESC_P2, 1);
                const uint64_t av = sw128_mnmajor_desc(sbase + PO_V + k * 2048, 8192, 1024);
                mma_f16_ss(tmem + 64, av, sw128_kmajor_desc(tb_u + k * 32), IDESC_P2, k != 0);
                mma_f16_ss(tmem + 64, av, sw128_kmajor_desc(tb_u + 8192 + k * 32), IDESC_P2, 1);
            }
            mma_commit(&m->bar_mma);
        }
        // the K̂ tile goes to the record while the MMAs run (the pass that
        // wrote it ended with a proxy fence and a barrier)
        if (tid == 0) {
            bulk_store(rec + REC_KH, sbase + PO_RT, 16384);
            bulk_commit();
        }
        if (!block_wait(&m->bar_mma, mph, &m->abort_flag, err, ERR_TIMEOUT_MMA)) break;
        mph ^= 1u;
        tc_fence_after();

        // ---- -W^T (fp16 high in RA, low in RX) and Ũ^T (fp16, RV and the
        //      record), thread = row d of W^T / r of Ũ^T, tokens half*32 .. +31 -----
        int sU = 0;
        {
            uint32_t x[32], y[32];
            tmem_ld32(tmem + lane_off + 0 + half * 32, x);
            tmem_ld32(tmem + lane_off + 64 + half * 32, y);
            tmem_wait_ld();
            float mw = 0.f, mu = 0.f;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                mw = fmaxf(mw, fabsf(__uint_as_float(x[e])));
                mu = fmaxf(mu, fabsf(__uint_as_float(y[e])));
            }
            block_scale2(mw, mu, m->red, sW, sU);
            const float fw = -exp2i(sW), fu = exp2i(sU);
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const uint32_t off = row * 128 + ((((half * 4 + c4) ^ (row & 7)) & 7) << 4);
                uint32_t hw[4], lw[4], hu[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = c4 * 8 + 2 * e;
                    f2h2_hilo(__uint_as_float(x[i]) * fw, __uint_as_float(x[i + 1]) * fw, hw[e], lw[e]);
                    hu[e] = f2h2_bits(__uint_as_float(y[i]) * fu, __uint_as_float(y[i + 1]) * fu);
                }
                smv4(sm, PO_RA + off, hw[0], hw[1], hw[2], hw[3]);
                smv4(sm, PO_RX + off, lw[0], lw[1], lw[2], lw[3]);
                smv4(sm, PO_V + off, hu[0], hu[1], hu[2], hu[3]);
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {   // Ũ^T is also the record's image
            bulk_store(rec + REC_UT, sbase + PO_V, 16384);
            bulk_commit();
        }

        // ---- N^T = K̂^T (-W) (columns 0-127) and P (-W) (rows 64-127 of
        //      columns 128-255), -W as fp16 high + low ------------------------------
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint64_t akh = sw128_mnmajor_desc(sbase + PO_RT + k * 2048, 8192, 1024);
                mma_f16_ss(tmem + 0, akh, sw128_kmajor_desc(sbase + PO_RA + k * 32), IDESC_NT, k != 0);
                mma_f16_ss(tmem + 0, akh, sw128_kmajor_desc(sbase + PO_RX + k * 32), IDESC_NT, 1);
                const uint64_t ap = sw128_kmajor_desc(sbase + PO_P - 8192 + k * 32);
                mma_f16_ss(tmem + 128, ap, sw128_kmajor_desc(sbase + PO_RA + k * 32), IDESC_H128, k != 0);
                mma_f16_ss(tmem + 128, ap, sw128_kmajor_desc(sbase + PO_RX + k * 32), IDESC_H128, 1);
            }
            mma_commit(&m->bar_mma);
        }
        if (!block_wait(&m->bar_mma, mph, &m->abort_flag, err, ERR_TIMEOUT_MMA)) break;
        mph ^= 1u;
        tc_fence_after();

        // ---- N^T (record, scale s_N): thread = row j, columns i = half*64 .. +63;
        //      Q' = Q̃ - P W (record, scale s_Q'): rows t = row - 64 --------------
        // Scales from bounds (every |operand| below 2^15 after its own scale):
        // |N| <= 64 2^30 2^-(s_K + s_W), |P W| <= 64 2^30 2^-(s_P + s_W),
        // |O⁰| <= 64 2^30 2^-(s_P + s_U); a bound above the true maximum only
        // moves values down within fp16's normal range.
        const int sN = min(max(sK + sW - 22, -100), 100);
        const int sQP = scale_exp(qbound + exp2c(36 - sP - sW));
        {
            const float gn = exp2c(sN - sK - sW), fpw = exp2i(-sP) * exp2i(-sW), gq = exp2i(sQP);
            const bool qrow = row >= C;            // warp-uniform (TMEM sub-partitions 2, 3)
            const int t = row - C;
            // Q̃ for columns half*64 + p*32 + 8*c8 .. +7 (p < 2, c8 < 4)
            auto qtilde = [&](int p, int c8, float (&qv)[8]) {
                const uint32_t a = PO_KQ + 8192 + half * 16384 + sw128_offset(t, p * 4 + c8);
                if (CHANNEL) {
                    const uint4 w = smv4(sm, a);
                    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
                    const float f = exp2i(-sQ);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 v = __half22float2(*reinterpret_cast<const __half2 *>(&ww[e]));
                        qv[2 * e] = v.x * f;
                        qv[2 * e + 1] = v.y * f;
                    }
                } else {
                    bf16x8_to_f32(smv4(sm, a), qv);
                    const float gq2 = m->u.s.gam[t];
#pragma unroll
                    for (int e = 0; e < 8; ++e) qv[e] *= gq2;
                }
            };
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                uint32_t x[32];
                tmem_ld32(tmem + lane_off + half * 64 + p * 32, x);
                tmem_wait_ld();
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        w[e] = f2h2_bits(__uint_as_float(x[c8 * 8 + 2 * e]) * gn,
                                         __uint_as_float(x[c8 * 8 + 2 * e + 1]) * gn);
                    smv4(sm, (half ? PO_RX : PO_RA) + row * 128 +
                                 ((((p * 4 + c8) ^ (row & 7)) & 7) << 4),
                         w[0], w[1], w[2], w[3]);
                }
                if (qrow) {
                    tmem_ld32(tmem + lane_off + 128 + half * 64 + p * 32, x);
                    tmem_wait_ld();
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) {
                        float qv[8];
                        qtilde(p, c8, qv);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            qv[e] = (qv[e] + __uint_as_float(x[c8 * 8 + e]) * fpw) * gq;
                        smv4(sm, PO_KQ + half * 16384 + t * 128 + ((((p * 4 + c8) ^ (t & 7)) & 7) << 4),
                             f2h2_bits(qv[0], qv[1]), f2h2_bits(qv[2], qv[3]),
                             f2h2_bits(qv[4], qv[5]), f2h2_bits(qv[6], qv[7]));
                    }
                }
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();   // TMEM columns 0-127 are read; N^T and Q' are staged
        if (tid == 0) {
            bulk_store(rec + REC_NT, sbase + PO_RA, 16384);
            bulk_store(rec + REC_NT + 16384, sbase + PO_RX, 16384);
            bulk_store(rec + REC_QP, sbase + PO_KQ, 8192);
            bulk_store(rec + REC_QP + 8192, sbase + PO_KQ + 16384, 8192);
            bulk_commit();
        }

        // ---- O⁰ = P Ũ (rows 64-127 of columns 0-127) ------------------------------
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_f16_ss(tmem + 0, sw128_kmajor_desc(sbase + PO_P - 8192 + k * 32),
                           sw128_kmajor_desc(sbase + PO_V + k * 32), IDESC_H128, k != 0);
            mma_commit(&m->bar_mma);
        }
        if (!block_wait(&m->bar_mma, mph, &m->abort_flag, err, ERR_TIMEOUT_MMA)) break;
        mph ^= 1u;
        tc_fence_after();
        {
            const int sO = min(max(sP + sU - 22, -100), 100);
            const float go = exp2c(sO - sP - sU);
            const int t = row - C;
            if (row >= C) {
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    uint32_t x[32];
                    tmem_ld32(tmem + lane_off + half * 64 + p * 32, x);
                    tmem_wait_ld();
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            w[e] = f2h2_bits(__uint_as_float(x[c8 * 8 + 2 * e]) * go,
                                             __uint_as_float(x[c8 * 8 + 2 * e + 1]) * go);
                        // rows 0-31 over Q d0-63, rows 32-63 over Q d64-127 (Q̃ is consumed)
                        smv4(sm, PO_KQ + 8192 + (t >> 5) * 16384 + (t & 31) * 256 +
                                     (half * 64 + p * 32 + c8 * 8) * 2,
                             w[0], w[1], w[2], w[3]);
                    }
                }
            }
            fence_proxy_async();
            __syncthreads();
            if (tid == 0) {
                bulk_store(rec + REC_OZ, sbase + PO_KQ + 8192, 8192);
                bulk_store(rec + REC_OZ + 8192, sbase + PO_KQ + 24576, 8192);
                bulk_commit();
                *reinterpret_cast<int4 *>(rec + REC_EX) = make_int4(sN, sK, sU, sQP);
                *reinterpret_cast<int4 *>(rec + REC_EX + 16) = make_int4(sO, 0, 0, 0);
            }
        }
    } while (0);
    // the record's bulk stores read this CTA's shared memory: they complete
    // before the CTA ends
    if (tid == 0) bulk_wait_all();

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, PREP_TMEM_COLS);
    }
}

// ----------------------------------------------------------- chain kernel ----
// One CTA per (sequence, head).  Per chunk, with S the state entering it:
//
//   MMA_B  D_B = Ũ^T K̂        A = record Ũ^T, B = record K̂ tile (MN-major);
//                              issued as soon as the last D_B was read
//   MMA_S  D_S = S N           A = S as fp16 high + low parts in TMEM, one
//                              power-of-two scale per row (value channel);
//                              B = record N^T
//   MMA_O  D_O = S Q'^T        A = the high part of S, B = record Q'
//
//   S' = S Diag(exp(G_C)) + D_S + D_B          (fp32, state warps)
//   O  = D_O^T + O⁰                             (output warps)
//
// MMA_S is the only product on the state's critical path: the state warps
// write the new S halves into TMEM and MMA_S of the next chunk starts.
// The high part of S alternates between two TMEM buffers, so the next
// chunk's state can be written while this chunk's MMA_O still reads it.
// Warps: 16 state warps (warp w: value channel r = 32 (w % 4) + lane, key
// channels 32 (w / 4) .. +31; the fp32 state lives in registers), 4 output
// warps (value channel r, all 64 tokens, through a shared-memory tile that
// leaves in 16-byte row segments), an MMA issuer and a record loader (two
// record stages, bulk copies, the records two chunks ahead prefetched to L2).
constexpr int kStateWarps = 16, kOutWarps = 4;
constexpr int kIssuerWarp = kStateWarps + kOutWarps, kLoaderWarp = kIssuerWarp + 1;
constexpr int kChainThreads = 32 * (kLoaderWarp + 1);   // 704
constexpr int kStateThreads = 32 * kStateWarps, kOutThreads = 32 * kOutWarps;
constexpr uint32_t CSTAGE = 99328;                       // record slot (1024-byte multiple)
constexpr uint32_t CO_OT = 2 * CSTAGE;                   // output tile [64 t][128 r] bf16
constexpr uint32_t CO_MISC = CO_OT + 16384;
constexpr uint32_t CHAIN_SMEM = CO_MISC + 8192;          // 223232
// TMEM: D_S, D_B, D_O, the high part of S in two buffers (chunk parity), the low part
constexpr uint32_t CT_DS = 0, CT_DB = 128, CT_DO = 256, CT_SH = 320, CT_SL = 448, CT_COLS = 512;
constexpr uint32_t IDESC_DB = make_idesc(0, 128, 128) | kIdescBMN;
static_assert(CHAIN_SMEM <= 232448 && REC_BYTES <= CSTAGE, "chain smem");

struct ChainMisc {
    uint64_t full[2], empty[2];       // record stage landed / free
    uint64_t bar_s, bar_o, bar_end;
    uint64_t s_hi, s_lo, d_free, o_free;      // S high / low part in TMEM
    uint32_t tmem_base;
    int abort_flag;
    int rowscale[4][D];               // S row exponents, by chunk mod 4
    float xs[2][4][D];                // row maxima of the four key-channel quarters, by chunk parity
};
static_assert(sizeof(ChainMisc) <= 8192, "chain misc area overflow");

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

__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <bool CHANNEL>
__global__ void __launch_bounds__(kChainThreads, 1)
chain_kernel(const uint8_t *__restrict__ recs, const float *h0, float *fin, float *ws_state,
             const int32_t *__restrict__ cu, int num_seqs, int total_T, int H, const ChunkMap map,
             __nv_bfloat16 *__restrict__ o, uint32_t *err) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = smem_u32(smem_raw);
    // segmented scan: which segment of which chain, and in which role
    // (0: the chain in full, 1: from a zero state without outputs, 2: the
    // transition from the identity, without B and outputs)
    int chain = blockIdx.x, seg = 0, role = 0;
    if (map.nseg > 0) {
        const int per = map.phase == 1 ? 2 * map.nseg - 3 : map.nseg - 1;
        chain = blockIdx.x / per;
        const int k = blockIdx.x % per;
        if (map.phase == 1) {
            seg = k == 0 ? 0 : 1 + (k - 1) / 2;
            role = k == 0 ? 0 : 1 + ((k - 1) & 1);
        } else {
            seg = 1 + k;
        }
    }
    const int h = chain % H, n = chain / H;
    int t0, len;
    sequence_range(cu, n, num_seqs, total_T, t0, len);
    const int b0 = map.base[n];
    const int nchunks = map.base[n + 1] - b0;
    const bool outputs = role == 0, use_b = role != 2, identity = role == 2;
    int c_begin, c_stop;
    const float *s_in;
    float *s_out;
    size_t in_off = 0, out_off = 0;
    if (map.nseg > 0) {
        const int L = (nchunks + map.nseg - 1) / map.nseg;
        c_begin = min(seg * L, nchunks);
        c_stop = min(c_begin + L, nchunks);
        auto slot = [&](int sg, int kind) { return (((size_t)chain * map.nseg + sg) * 3 + kind) * D * D; };
        s_in = role != 0 ? nullptr : (seg == 0 ? h0 : map.slots);
        in_off = seg == 0 ? (size_t)chain * D * D : slot(seg, 0);
        if (map.phase == 1) {
            s_out = map.slots;
            out_off = role == 0 ? slot(1, 0) : slot(seg, role);
        } else {
            s_out = seg == map.nseg - 1 ? fin : nullptr;
            out_off = (size_t)chain * D * D;
        }
    } else {
        // this launch's local chunks of the sequence
        c_begin = max(map.c0, map.w0 - b0);
        c_stop = min(min(map.c1, map.w1 - b0), nchunks);
        const bool first_launch = map.c0 == 0 && map.w0 == 0;
        if (c_stop <= c_begin && !(nchunks == 0 && first_launch)) return;   // nothing here
        // the state enters from the initial state or from the launch before; it
        // leaves to the final state or to the launch after (pieces: one slot per
        // chain; windows: one slot per window boundary, which one sequence crosses)
        const size_t slot_in = map.by_window ? ((size_t)(map.win - 1) * H + h) : (size_t)chain;
        const size_t slot_out = map.by_window ? ((size_t)map.win * H + h) : (size_t)chain;
        s_in = c_begin == 0 ? h0 : ws_state;
        s_out = c_stop == nchunks ? fin : ws_state;
        in_off = (c_begin == 0 ? (size_t)chain : slot_in) * D * D;
        out_off = (c_stop == nchunks ? (size_t)chain : slot_out) * D * D;
    }
    const int nl = max(c_stop - c_begin, 0);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int sub = warp & 3;                          // TMEM sub-partition of this warp
    const int r = sub * 32 + lane;                     // value channel = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(sub * 32) << 16;
    const int qc = (warp >> 2) & 3;                    // state warps: key-channel quarter
    const size_t tsg = (size_t)r * D + qc * 32;   // this thread's part of a state

    if (nl == 0) {   // no chunks: the state (or the identity) passes through
        if (s_out != nullptr && warp < kStateWarps) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                if (s_in != nullptr) x = *reinterpret_cast<const float4 *>(s_in + in_off + tsg + j);
                if (identity) {
                    x.x = r == qc * 32 + j ? 1.f : 0.f;
                    x.y = r == qc * 32 + j + 1 ? 1.f : 0.f;
                    x.z = r == qc * 32 + j + 2 ? 1.f : 0.f;
                    x.w = r == qc * 32 + j + 3 ? 1.f : 0.f;
                }
                *reinterpret_cast<float4 *>(s_out + out_off + tsg + j) = x;
            }
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
        for (int s = 0; s < 2; ++s) {
            mbar_init(&m->full[s], 1);
            mbar_init(&m->empty[s], 1 + kStateThreads + (outputs ? kOutThreads : 0));
        }
        mbar_init(&m->bar_s, 1);
        mbar_init(&m->bar_o, 1);
        mbar_init(&m->o_free, kOutThreads);
        mbar_init(&m->bar_end, 1);
        mbar_init(&m->s_hi, kStateThreads);
        mbar_init(&m->s_lo, kStateThreads);
        mbar_init(&m->d_free, kStateThreads);
        m->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&m->tmem_base, CT_COLS);
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
        return recs + ((size_t)(b0 + c_begin + lc - map.w0) * H + h) * REC_BYTES;
    };

    if (warp < kStateWarps) {
        // ========= state warps: value channel r, key channels qc*32 .. +31 ========
        float S[32];
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (s_in != nullptr) x = *reinterpret_cast<const float4 *>(s_in + in_off + tsg + j);
            S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
        }
        if (identity) {
#pragma unroll
            for (int j = 0; j < 32; ++j) S[j] = r == qc * 32 + j ? 1.f : 0.f;
        }
        bool stop = false;
        // S entering chunk lc -> fp16 high and low parts in TMEM with the row's
        // own scale (the four quarters of a row agree on it through the
        // barrier, which also agrees on stopping)
        auto publish = [&](int lc) {
            float mx = 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) mx = fmaxf(mx, fabsf(S[j]));
            m->xs[lc & 1][qc][r] = mx;
            stop = named_sync_or(1, kStateThreads, stop || *abort_flag != 0);
#pragma unroll
            for (int k = 0; k < 4; ++k) mx = fmaxf(mx, m->xs[lc & 1][k][r]);
            const int s = scale_exp(mx);
            const float f = exp2i(s);
            // the high part goes first: its MMAs start while the low part is stored
            uint32_t hi[16], lo[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) hi[jj] = f2h2_bits(S[2 * jj] * f, S[2 * jj + 1] * f);
            tmem_st16(tmem + lane_off + CT_SH + (lc & 1) * 64 + qc * 16, hi);
            tmem_wait_st();
            if (qc == 0) m->rowscale[lc & 3][r] = s;
            tc_fence_before();
            mbar_arrive(&m->s_hi);
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const float2 hv = __half22float2(*reinterpret_cast<const __half2 *>(&hi[jj]));
                lo[jj] = f2h2_bits(fmaf(S[2 * jj], f, -hv.x), fmaf(S[2 * jj + 1], f, -hv.y));
            }
            tmem_st16(tmem + lane_off + CT_SL + qc * 16, lo);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&m->s_lo);
            return s;
        };
        int sS = publish(0);
        for (int lc = 0; lc < nl && !stop; ++lc) {
            const uint32_t s = lc & 1;
            const uint8_t *stg = sm + s * CSTAGE;
            if (!warp_wait(&m->full[s], (lc >> 1) & 1)) { fail(ERR_TIMEOUT_TMA); stop = true; }
            if (!stop && !warp_wait(&m->bar_s, lc & 1)) { fail(ERR_TIMEOUT_MMA); stop = true; }
            if (!stop) {
                tc_fence_after();
                const int *ex = reinterpret_cast<const int *>(stg + REC_EX);
                const float fs = exp2i(-sS) * exp2i(-ex[0]), fb = exp2i(-ex[2]) * exp2i(-ex[1]);
                const float *gc = reinterpret_cast<const float *>(stg + REC_GC) + (CHANNEL ? qc * 32 : 0);
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    uint32_t xd[16], xb[16];
                    tmem_ld16(tmem + lane_off + CT_DS + qc * 32 + p * 16, xd);
                    if (use_b) {
                        tmem_ld16(tmem + lane_off + CT_DB + qc * 32 + p * 16, xb);
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) xb[e] = 0u;
                    }
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int j = p * 16 + e;
                        const float gcj = CHANNEL ? gc[j] : gc[0];
                        S[j] = fmaf(gcj, S[j],
                                    fmaf(__uint_as_float(xd[e]), fs, __uint_as_float(xb[e]) * fb));
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&m->d_free);     // D_S and D_B are read
            mbar_arrive(&m->empty[s]);   // this stage's gates and exponents are read
            // S entering chunk lc + 1: its high part goes to the buffer that
            // chunk lc - 1 read.  This chunk's MMA_O may still read the other one;
            // MMA_S and MMA_O of chunk lc - 1 were issued before the commit of
            // bar_s above, so they are complete.
            if (lc + 1 < nl) sS = publish(lc + 1);
        }
        if (s_out != nullptr) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<float4 *>(s_out + out_off + tsg + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    } else if (warp < kIssuerWarp) {
        // ================== output warps: value channel r, all 64 tokens ==========
        const int otid = tid - kStateThreads;
        bool stop = false;
        for (int lc = 0; lc < (outputs ? nl : 0); ++lc) {
            const uint32_t s = lc & 1;
            const uint8_t *stg = sm + s * CSTAGE;
            // take this chunk's O⁰ column r and exponents, then free the record
            // stage at once, so the loader can refill it early
            if (!warp_wait(&m->full[s], (lc >> 1) & 1)) { fail(ERR_TIMEOUT_TMA); stop = true; }
            uint32_t zp[32];
            int eq = 0, eo = 0;
            if (!stop) {
                const uint16_t *oz = reinterpret_cast<const uint16_t *>(stg + REC_OZ) + r;
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    zp[e] = (uint32_t)oz[(2 * e) * 128] | ((uint32_t)oz[(2 * e + 1) * 128] << 16);
                const int *ex = reinterpret_cast<const int *>(stg + REC_EX);
                eq = ex[3];
                eo = ex[4];
            }
            mbar_arrive(&m->empty[s]);
            if (!stop && !warp_wait(&m->bar_o, lc & 1)) { fail(ERR_TIMEOUT_MMA); stop = true; }
            if (!stop) {
                tc_fence_after();
                const float fo = exp2i(-m->rowscale[lc & 3][r]) * exp2i(-eq), fz = exp2i(-eo);
                __nv_bfloat16 *tile = reinterpret_cast<__nv_bfloat16 *>(sm + CO_OT) + r;
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    uint32_t x[16];
                    tmem_ld16(tmem + lane_off + CT_DO + p * 16, x);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; e += 2) {
                        const float2 z = __half22float2(*reinterpret_cast<const __half2 *>(&zp[(p * 16 + e) / 2]));
                        tile[(p * 16 + e) * 128] = __float2bfloat16_rn(fmaf(__uint_as_float(x[e]), fo, z.x * fz));
                        tile[(p * 16 + e + 1) * 128] =
                            __float2bfloat16_rn(fmaf(__uint_as_float(x[e + 1]), fo, z.y * fz));
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&m->o_free);
            stop = named_sync_or(3, kOutThreads, stop || *abort_flag != 0);
            if (stop) break;
            {   // 64 rows x 256 bytes leave as 16-byte segments; rows past the end stay
                const int cc = c_begin + lc;
                const int cl = min(C, len - cc * C);
                const uint4 *tile = reinterpret_cast<const uint4 *>(sm + CO_OT);
#pragma unroll
                for (int q = 0; q < 1024 / kOutThreads; ++q) {
                    const int e = q * kOutThreads + otid;   // row e / 16, segment e % 16
                    const int i = e >> 4, seg = e & 15;
                    if (i < cl)
                        *reinterpret_cast<uint4 *>(o + ((size_t)(t0 + cc * C + i) * H + h) * D + seg * 8) = tile[e];
                }
            }
            named_sync(3, kOutThreads);   // the tile is free again
        }
    } else if (warp == kIssuerWarp) {
        // ======================================================= MMA issuer ====
        if (lane == 0) {
            for (int lc = 0; lc < nl; ++lc) {
                if (*abort_flag) break;
                const uint32_t s = lc & 1;
                const uint32_t stg = sbase + s * CSTAGE;
                if (!mbar_wait_sleep(&m->full[s], (lc >> 1) & 1)) { fail(ERR_TIMEOUT_TMA); break; }
                if (lc > 0 && !mbar_wait_sleep(&m->d_free, (lc - 1) & 1)) { fail(ERR_TIMEOUT_HANDOFF); break; }
                tc_fence_after();
                if (use_b) {
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_f16_ss(tmem + CT_DB, sw128_kmajor_desc(stg + REC_UT + k * 32),
                                   sw128_mnmajor_desc(stg + REC_KH + k * 2048, 8192, 1024), IDESC_DB, k != 0);
                }
                if (!mbar_wait_sleep(&m->s_hi, lc & 1)) { fail(ERR_TIMEOUT_HANDOFF); break; }
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_f16_ts(tmem + CT_DS, tmem + CT_SH + s * 64 + k * 8,
                               sw128_kmajor_desc(stg + REC_NT + (k >> 2) * 16384 + (k & 3) * 32),
                               IDESC_H128, k != 0);
                if (!mbar_wait_sleep(&m->s_lo, lc & 1)) { fail(ERR_TIMEOUT_HANDOFF); break; }
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_f16_ts(tmem + CT_DS, tmem + CT_SL + k * 8,
                               sw128_kmajor_desc(stg + REC_NT + (k >> 2) * 16384 + (k & 3) * 32),
                               IDESC_H128, 1);
                mma_commit(&m->bar_s);
                if (!outputs) {
                    mma_commit(&m->empty[s]);
                    continue;
                }
                if (lc >= 1 && !mbar_wait_sleep(&m->o_free, (lc - 1) & 1)) {
                    fail(ERR_TIMEOUT_HANDOFF);
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_f16_ts(tmem + CT_DO, tmem + CT_SH + s * 64 + k * 8,
                               sw128_kmajor_desc(stg + REC_QP + (k >> 2) * 8192 + (k & 3) * 32),
                               IDESC_H64, k != 0);
                mma_commit(&m->bar_o);
                mma_commit(&m->empty[s]);
            }
            // every MMA issued here is complete before TMEM is freed
            mma_commit(&m->bar_end);
            (void)mbar_wait_sleep(&m->bar_end, 0);
        }
    } else if (lane == 0) {
        // ==================================================== record loader ====
        uint32_t issued[2] = {0, 0};
        for (int lc = 0; lc < nl; ++lc) {
            if (*abort_flag) break;
            const int s = lc & 1;
            if (lc >= 2 && !mbar_wait_sleep(&m->empty[s], ((lc - 2) >> 1) & 1)) {
                fail(ERR_TIMEOUT_HANDOFF);
                break;
            }
            mbar_arrive_expect_tx(&m->full[s], REC_BYTES);
            bulk_load(sm + s * CSTAGE, rec_of(lc), REC_BYTES, &m->full[s]);
            ++issued[s];
            if (lc + 2 < nl) {
                const uint8_t *pr = rec_of(lc + 2);
                bulk_prefetch_l2(pr, REC_BYTES / 2);
                bulk_prefetch_l2(pr + REC_BYTES / 2, REC_BYTES / 2);
            }
        }
        // never leave a bulk copy in flight into this CTA's shared memory
        for (int s = 0; s < 2; ++s)
            if (issued[s] > 0) (void)mbar_wait_sleep(&m->full[s], (issued[s] - 1) & 1);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, CT_COLS);
    }
}

// ------------------------------------------------------------------ host ----

constexpr size_t kHeaderBytes = 256;                        // error word
constexpr size_t kMaxRecordBytes = size_t(8) << 30;         // records per window
// Pipelined pieces need the chain CTAs to leave most SMs to the prep kernel;
// beyond this many (sequence, head) chains the plan runs the prep kernel over
// a whole window first, then the chain kernel.
constexpr int kPipeChains = 64;
// Segmented scan: at most this many segments per sequence, and phase-1 CTAs
// (2 per segment) within about one per SM.
constexpr int kMaxSegments = 8, kSegCTAs = 148;

struct SplitPlan {
    int chains = 0, max_chunks = 0;
    long long max_total = 0;        // bound on the number of global chunks
    int window = 0, windows = 0;    // global chunks per window, windows
    int pieces = 1;                 // pipeline pieces of a single window
    int nseg = 0;                   // segments per sequence of the segmented scan
    bool by_window = false;
    size_t base_off = 0, state_off = 0, rec_off = 0, bytes = 0;
};

// Pipeline pieces of one window: the prep kernel of piece k + 1 runs beside
// the chain kernel of piece k; each piece is 1.3 times the one before:
// 12, 16, 21, 27, 35, ... chunks, the last one the remainder.  Writes the
// piece boundaries (count + 1 of them) and returns the count.
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
// tokens; otherwise the lengths live on the device, and the number of
// chunks of all sequences together is at most total_T / 64 + num_seqs.
bool make_split_plan(int num_seqs, int total_T, int H, SplitPlan &p, bool equal_lengths = false) {
    const long long chains = (long long)num_seqs * H;
    if (chains < 1 || chains > (1ll << 24) || total_T <= 0) return false;
    p.chains = (int)chains;
    const int longest = equal_lengths ? total_T / num_seqs : total_T;
    p.max_chunks = (longest + C - 1) / C;   // no sequence has more chunks
    p.max_total = equal_lengths ? (long long)num_seqs * p.max_chunks
                                : (long long)(total_T + C - 1) / C + num_seqs;
    const size_t per = (size_t)H * REC_BYTES;
    const long long fit = (long long)(kMaxRecordBytes / per);
    if (fit < 1) return false;
    p.window = (int)std::min(p.max_total, fit);
    p.windows = (int)((p.max_total + p.window - 1) / p.window);
    int bounds[kMaxPieces + 1];
    p.by_window = !(p.windows == 1 && chains <= kPipeChains);
    p.pieces = p.by_window ? 1 : piece_schedule(p.max_chunks, bounds);
    // Few chains: the segmented scan, sized so that its first phase (one CTA
    // for the first segment, two for each later one but the last:
    // chains (2 nseg - 3) CTAs) fits the 148 SMs at once
    if (!p.by_window) {
        const int ns = std::min(kMaxSegments, (kSegCTAs / p.chains + 3) / 2);
        if (ns >= 3 && p.max_chunks >= 2 * ns) {
            p.nseg = ns;
            p.pieces = 1;
        }
    }
    size_t state = 0;   // slots for states between launches
    if (p.by_window) state = (size_t)(p.windows - 1) * H * D * D * sizeof(float);
    else if (p.nseg > 0) state = (size_t)p.chains * p.nseg * 3 * D * D * sizeof(float);
    else if (p.pieces > 1) state = (size_t)p.chains * D * D * sizeof(float);
    p.base_off = kHeaderBytes;
    p.state_off = (p.base_off + (size_t)(num_seqs + 1) * sizeof(int32_t) + 255) & ~size_t(255);
    p.rec_off = (p.state_off + state + 1023) & ~size_t(1023);
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

}  // namespace

size_t tcgen05_split_workspace_bytes(int num_seqs, int total_T, int H) {
    // the caller may pass cu_seqlens or not: room for either plan
    SplitPlan p, pe;
    if (!make_split_plan(num_seqs, total_T, H, p)) return 0;
    const bool equal_ok = total_T % num_seqs == 0 && make_split_plan(num_seqs, total_T, H, pe, true);
    return equal_ok ? std::max(p.bytes, pe.bytes) : p.bytes;
}

cudaError_t launch_prefill_split(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const float *h0, const int32_t *cu,
                                 int num_seqs, int total_T, int Hqk, int H, bool channel, void *o,
                                 float *fin, void *workspace, cudaStream_t stream,
                                 const PrologueIn *pin) {
    SplitPlan p;
    if (!make_split_plan(num_seqs, total_T, H, p, cu == nullptr)) return cudaErrorInvalidValue;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint32_t *err = reinterpret_cast<uint32_t *>(ws);
    int32_t *base = reinterpret_cast<int32_t *>(ws + p.base_off);
    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(uint32_t), stream);
    if (e != cudaSuccess) return e;
    // with the fused prologue the tiles are computed, not loaded: the maps
    // (over the raw projections, of the same shape) are passed but unused
    const bool fused = pin != nullptr;
    PrologueIn pi = {};
    if (fused) {
        pi = *pin;
        q = pi.xq;
        k = pi.xk;
        v = pi.xv;
    }
    CUtensorMap mq, mk, mv, mg;
    if (!make_map(&mq, q, total_T, Hqk) || !make_map(&mk, k, total_T, Hqk) ||
        !make_map(&mv, v, total_T, H))
        return cudaErrorInvalidValue;
    if (channel && !fused) {
        if (!make_gate_map(&mg, g, total_T, H)) return cudaErrorInvalidValue;
    } else {
        mg = mq;   // not read
    }
    auto prep = channel ? (fused ? prep_kernel<true, true> : prep_kernel<true, false>)
                        : (fused ? prep_kernel<false, true> : prep_kernel<false, false>);
    e = ensure_dynamic_smem(reinterpret_cast<const void *>(prep), (int)PREP_SMEM);
    if (e != cudaSuccess) return e;
    auto chain_k = channel ? chain_kernel<true> : chain_kernel<false>;
    e = ensure_dynamic_smem(reinterpret_cast<const void *>(chain_k), (int)CHAIN_SMEM);
    if (e != cudaSuccess) return e;
    float *state = reinterpret_cast<float *>(ws + p.state_off);
    uint8_t *recs = ws + p.rec_off;
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(o);
    chunk_base_kernel<<<1, 1024, 0, stream>>>(cu, num_seqs, total_T, base);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    auto run_chain = [&](const ChunkMap &map, cudaStream_t st) {
        chain_k<<<(unsigned)p.chains, kChainThreads, CHAIN_SMEM, st>>>(recs, h0, fin, state, cu, num_seqs,
                                                                        total_T, H, map, out, err);
        return cudaGetLastError();
    };
    auto run_prep = [&](const ChunkMap &map, unsigned gx, unsigned gy, cudaStream_t st) {
        prep<<<dim3(gx, gy), kPrepThreads, PREP_SMEM, st>>>(mq, mk, mv, mg, g, beta, cu, num_seqs, total_T,
                                                            Hqk, H, map, recs, pi, err);
        return cudaGetLastError();
    };
    constexpr int kAll = 1 << 30;
    if (p.nseg > 0) {
        // the prep kernel over every chunk, then the segmented scan
        const ChunkMap all{base, 0, (int)p.max_total, 0, p.max_chunks, 0, 0};
        e = run_prep(all, (unsigned)p.max_chunks, (unsigned)p.chains, stream);
        if (e != cudaSuccess) return e;
        ChunkMap seg{base, 0, (int)p.max_total, 0, kAll, 0, 0, p.nseg, 1, state};
        chain_k<<<(unsigned)(p.chains * (2 * p.nseg - 3)), kChainThreads, CHAIN_SMEM, stream>>>(
            recs, h0, fin, state, cu, num_seqs, total_T, H, seg, out, err);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        e = ensure_dynamic_smem(reinterpret_cast<const void *>(segment_compose_kernel), (int)COMPOSE_SMEM);
        if (e != cudaSuccess) return e;
        segment_compose_kernel<<<dim3((unsigned)p.chains, D / 16), kComposeThreads, COMPOSE_SMEM, stream>>>(
            state, p.nseg);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        seg.phase = 2;
        chain_k<<<(unsigned)(p.chains * (p.nseg - 1)), kChainThreads, CHAIN_SMEM, stream>>>(
            recs, h0, fin, state, cu, num_seqs, total_T, H, seg, out, err);
        return cudaGetLastError();
    }
    if (!p.by_window) {
        // one window holds every record; pieces of every sequence's chunks
        int bounds[kMaxPieces + 1];
        piece_schedule(p.max_chunks, bounds);
        auto piece = [&](int k) {
            // w1 = the records' capacity: a malformed cu_seqlens with more chunks
            // than total_T allows never writes past it
            return ChunkMap{base, 0, (int)p.max_total, bounds[k], bounds[k + 1], 0, 0};
        };
        if (p.pieces == 1) {
            e = run_prep(piece(0), (unsigned)(bounds[1] - bounds[0]), (unsigned)p.chains, stream);
            return e == cudaSuccess ? run_chain(piece(0), stream) : e;
        }
        // the prep kernel of piece k + 1 runs on the SMs the chain kernel of
        // piece k leaves free
        std::lock_guard<std::mutex> lock(g_helpers_mutex);
        Helpers *hs = nullptr;
        e = get_helpers(&hs);
        if (e != cudaSuccess) return e;
        e = cudaEventRecord(hs->fork, stream);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(hs->prep_s, hs->fork, 0);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(hs->chain_s, hs->fork, 0);
        for (int kk = 0; kk < p.pieces && e == cudaSuccess; ++kk) {
            e = run_prep(piece(kk), (unsigned)(bounds[kk + 1] - bounds[kk]), (unsigned)p.chains, hs->prep_s);
            if (e == cudaSuccess) e = cudaEventRecord(hs->prep_done, hs->prep_s);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(hs->chain_s, hs->prep_done, 0);
            if (e == cudaSuccess) e = run_chain(piece(kk), hs->chain_s);
        }
        if (e == cudaSuccess) e = cudaEventRecord(hs->join, hs->chain_s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, hs->join, 0);
        return e;
    }
    // windows of global chunks: the prep kernel over a window, then the chain
    for (int w = 0; w < p.windows; ++w) {
        const long long w0 = (long long)w * p.window;
        const long long w1 = std::min(w0 + p.window, p.max_total);
        const ChunkMap map{base, (int)w0, (int)w1, 0, kAll, w, 1};
        e = run_prep(map, (unsigned)(w1 - w0), (unsigned)H, stream);
        if (e != cudaSuccess) return e;
        e = run_chain(map, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace gdr
