// Gradient of the recurrence in chunked form (scalar gate, d_k = d_v = 128):
// the chunk algebra of the prefill (page "How the New Flash Models Work:
// Inside GLM-5.3-Flash and Qwen3.8-Flash-Next", section "Linear attention: a
// fixed-size memory in place of the cache", rearranged per chunk of C = 64
// tokens) run backwards.  Per chunk, with S the state entering it, G the
// chunk-cumulative log-gate, gamma = e^G and R_ij = e^{G_i - G_j}:
//
//   A = strictly-lower(diag(beta) (K K^T) o R),  T = (I + A)^-1
//   W = T diag(beta gamma) K,  U~ = T diag(beta) V,  U = U~ - W S^T
//   P = causal((Q K^T) o R),  O = diag(gamma) Q S^T + P U
//   S' = e^{G_C} S + U^T K^,   K^_j = k_j e^{G_C - G_j}
//
// With L' the adjoint of S' (dS_final after a sequence's last chunk), the
// adjoint of the state entering the chunk is
//
//   dU = K^ L'^T + P^T dO,   L = e^{G_C} L' + dO^T diag(gamma) Q - dU^T W
//
// and the chunk-local gradients follow from S, L', dO and the chunk's own
// quantities: dK^ = U L', dW = -dU S, dP = causal(dO U^T), d(gamma Q) = dO S,
// dT = dU (beta V)^T + dW (beta gamma K)^T, dA = -T^T dT T^T (strictly
// lower), and from these dq, dk, dv, dbeta and the adjoints of G, whose
// reverse cumulative sum within the chunk is dg.  Four launches:
//
//   chunk base  the first global chunk of every sequence.
//   prep        one CTA per (chunk, head): A, T, W, U~, P, K^, diag(gamma) Q,
//               G, beta and the upstream terms of the adjoint chain,
//               Y = dO^T diag(gamma) Q and Z = P^T dO (fp32 record).
//   chains      one CTA of 512 threads per (sequence, head, 16 state rows):
//               warps 0-7 carry the state forward (S and U of every chunk),
//               warps 8-15 the adjoint backward (L' and dU = Z + K^ L'^T of
//               every chunk, L = e^{G_C} L' + Y - dU^T W, the adjoint of the
//               initial state at the end).
//   local       one CTA per (chunk, head): every gradient of the chunk's
//               tokens.
//
// Every product runs on the tensor cores as warp-level MMAs over operands
// split into a high and a low part (bf16, or tf32 for K K^T and Q K^T), in up
// to three passes with fp32 accumulation (see the products below).  The chunk records live in the workspace: 475,648 bytes per
// (chunk, head).
#include <cuda_bf16.h>

#include <algorithm>
#include <cstddef>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "chunk_common.cuh"
#include "tc_ptx.cuh"

namespace gdr {
namespace {

// per (chunk, head) record of floats
constexpr size_t R_W = 0;                       // W [64][128]
constexpr size_t R_UT = R_W + C * D;            // U~ [64][128]
constexpr size_t R_P = R_UT + C * D;            // P^T [64][64] (P causal)
constexpr size_t R_T = R_P + C * C;             // T [64][64], lower with the unit diagonal
constexpr size_t R_AR = R_T + C * C;            // (K K^T) o R [64][64], strictly lower
constexpr size_t R_G = R_AR + C * C;            // G [64] (the chunk's cumulative log-gate)
constexpr size_t R_B = R_G + C;                 // beta [64] (0 past the sequence's end)
constexpr size_t R_U = R_B + C;                 // U [64][128]
constexpr size_t R_DU = R_U + C * D;            // dU [64][128]
constexpr size_t R_S = R_DU + C * D;            // state entering the chunk [128][128]
constexpr size_t R_L = R_S + D * D;             // adjoint of the state leaving it [128][128]
constexpr size_t R_KH = R_L + D * D;            // K^ [64][128]
constexpr size_t R_QT = R_KH + C * D;           // diag(gamma) Q [64][128]
constexpr size_t R_Y = R_QT + C * D;            // dO^T diag(gamma) Q [128][128]
constexpr size_t R_Z = R_Y + D * D;             // P^T dO [64][128]
constexpr size_t R_FLOATS = R_Z + C * D;        // 118,912 floats
constexpr size_t kBaseBytes = 256;              // sequence chunk offsets precede the records

constexpr int LW = D + 4;    // padded row of 128 floats (4 mod 32: see the products)
constexpr int LN = C + 4;    // padded row of 64 floats
constexpr int kRowBlock = 16;                   // state rows per forward / reverse CTA
constexpr int kLocalThreads = 256;
constexpr int kLocTM = 4, kLocTN = 8;   // slots of a thread in a <C, D> product over 8 warps

// ---------------------------------------------------- tensor-core products ----
// An input held as bf16 is exact in tf32.
template <typename IoT> constexpr bool kIoExact = std::is_same<IoT, __nv_bfloat16>::value;

// Products in fp32 accuracy on the tensor cores: each operand value x is
// split into x_hi = tf32(x) and x_lo = tf32(x - x_hi), and the product is
// accumulated in fp32 as lo*hi + hi*lo + hi*hi (the dropped lo*lo term is
// below 2^-21 of it).  Warp-level m16n8k8 tf32 tiles whose fragments are
// read from shared memory through the accessors a(m, k) and b(k, n), so a
// stored matrix serves in either orientation; rows padded to 4 mod 32 floats
// keep every fragment read within two-way bank conflicts.

__device__ __forceinline__ void split_tf32(float x, uint32_t &hi, uint32_t &lo) {
    hi = tc::to_tf32(x);
    lo = tc::to_tf32(x - __uint_as_float(hi));
}

// d (16 x 8, fp32) += a (16 x 8, tf32, row) * b (8 x 8, tf32, column).
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// How NW warps share an M x N result: GM x GN warp blocks of WM x WN, each
// MT x NT tiles of 16 x 8.
template <int M, int N, int NW>
struct WarpGrid {
    static constexpr int pick() {
        return (M % 32 == 0 && NW % 2 == 0 && N % (8 * (NW / 2)) == 0)   ? 2
               : (M % 64 == 0 && NW % 4 == 0 && N % (8 * (NW / 4)) == 0) ? 4
                                                                          : 1;
    }
    static constexpr int GM = pick(), GN = NW / GM;
    static constexpr int WM = M / GM, WN = N / GN;
    static constexpr int MT = WM / 16, NT = WN / 8;
    static_assert(GM * GN == NW && MT * 16 * GM == M && NT * 8 * GN == N, "warp tiling");
};

// out(m, n) = sum_k a(m, k) b(k, n) over NTH threads (K a multiple of 8);
// every result goes to epi(r, c, m, n, value) with (r, c) its slot in the
// calling thread's part (r < 2 MT, c < 2 NT).  Every <M, N, NTH> product
// hands a thread the same (m, n) in the same slot, so that a caller can sum
// several products in registers.  AEX (BEX) states that every value a (b)
// returns is exact in tf32 (a bf16 input), so that its low part and the pass
// that multiplies it are skipped.
template <int M, int N, int NTH, bool AEX = false, bool BEX = false, class AF, class BF, class EPI>
__device__ __forceinline__ void tgemm_rc(int K, AF a, BF b, EPI epi) {
    using G = WarpGrid<M, N, NTH / 32>;
    const int t = threadIdx.x & (NTH - 1), lane = t & 31, warp = t >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    const int m0 = (warp / G::GN) * G::WM, n0 = (warp % G::GN) * G::WN;
    float acc[G::MT][G::NT][4];
#pragma unroll
    for (int mt = 0; mt < G::MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < G::NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
    auto take = [](float x, uint32_t &hi, uint32_t &lo, bool exact) {
        if (exact) hi = __float_as_uint(x);
        else split_tf32(x, hi, lo);
    };
#pragma unroll 2
    for (int k0 = 0; k0 < K; k0 += 8) {
        uint32_t ah[G::MT][4], al[G::MT][4], bh[G::NT][2], bl[G::NT][2];
#pragma unroll
        for (int mt = 0; mt < G::MT; ++mt) {
            const int m = m0 + mt * 16 + gid;
            take(a(m, k0 + tig), ah[mt][0], al[mt][0], AEX);
            take(a(m + 8, k0 + tig), ah[mt][1], al[mt][1], AEX);
            take(a(m, k0 + tig + 4), ah[mt][2], al[mt][2], AEX);
            take(a(m + 8, k0 + tig + 4), ah[mt][3], al[mt][3], AEX);
        }
#pragma unroll
        for (int nt = 0; nt < G::NT; ++nt) {
            const int n = n0 + nt * 8 + gid;
            take(b(k0 + tig, n), bh[nt][0], bl[nt][0], BEX);
            take(b(k0 + tig + 4, n), bh[nt][1], bl[nt][1], BEX);
        }
#pragma unroll
        for (int mt = 0; mt < G::MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < G::NT; ++nt) {
                if (!AEX) mma_tf32(acc[mt][nt], al[mt], bh[nt]);
                if (!BEX) mma_tf32(acc[mt][nt], ah[mt], bl[nt]);
                mma_tf32(acc[mt][nt], ah[mt], bh[nt]);
            }
    }
#pragma unroll
    for (int mt = 0; mt < G::MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < G::NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                epi(mt * 2 + (e >> 1), nt * 2 + (e & 1), m0 + mt * 16 + gid + 8 * (e >> 1),
                    n0 + nt * 8 + 2 * tig + (e & 1), acc[mt][nt][e]);
}

template <int M, int N, int NTH, bool AEX = false, bool BEX = false, class AF, class BF, class EPI>
__device__ __forceinline__ void tgemm(int K, AF a, BF b, EPI epi) {
    tgemm_rc<M, N, NTH, AEX, BEX>(K, a, b, [&](int, int, int m, int n, float v) { epi(m, n, v); });
}

// The same products in bf16: each value x splits into x_hi = bf16(x) and
// x_lo = bf16(x - x_hi) (16 significant bits together, the fp32 exponent
// range), accumulated in fp32 as lo*hi + hi*lo + hi*hi with m16n8k16 MMAs
// (twice the k-depth of a tf32 MMA per instruction).  Each product term is
// off by about 2^-16 of its size, which the chunk-local gradients (one
// product deep, nothing carried from chunk to chunk) can take; the chains
// keep the tf32 form.  AEX / BEX as above (a bf16 input is exact).

__device__ __forceinline__ uint32_t pack_bf16(float lo_elem, float hi_elem) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo_elem, hi_elem);
    return *reinterpret_cast<const uint32_t *>(&p);
}
// Two values -> their high pair and low pair.
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t &hi, uint32_t &lo) {
    hi = pack_bf16(x0, x1);
    const float h0 = __uint_as_float(hi << 16), h1 = __uint_as_float(hi & 0xFFFF0000u);
    lo = pack_bf16(x0 - h0, x1 - h1);
}

// d (16 x 8, fp32) += a (16 x 16, bf16, row) * b (16 x 8, bf16, column).
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// tgemm_rc's contract with bf16 products; K a multiple of 16 KPAR.
//   PAIRS: the results go out two at a time, epi(r, m, n, value(m, n),
//          value(m, n + 1)) with n even and r the row's slot, so that a
//          store can take both.
//   KPAR, PSPLIT: a warp with few tiles would wait on one long chain of
//          dependent MMAs, so KPAR = 2 alternates the k-steps between two
//          sets of accumulators and PSPLIT gives each pass its own set, the
//          sets summed at the end.
//   APAIR, BPAIR: the accessor returns the k-pair (x(k), x(k + 1)) for even
//          k as a float2 (one 8-byte load from a k-contiguous row).
template <int M, int N, int NTH, bool AEX = false, bool BEX = false, bool PAIRS = false,
          int KPAR = 1, bool PSPLIT = false, bool APAIR = false, bool BPAIR = false, class AF,
          class BF, class EPI>
__device__ __forceinline__ void bgemm_rc(int K, AF a, BF b, EPI epi) {
    using G = WarpGrid<M, N, NTH / 32>;
    constexpr int NP = PSPLIT ? 3 : 1;
    const int t = threadIdx.x & (NTH - 1), lane = t & 31, warp = t >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    const int m0 = (warp / G::GN) * G::WM, n0 = (warp % G::GN) * G::WN;
    float acc[KPAR][NP][G::MT][G::NT][4];
#pragma unroll
    for (int s = 0; s < KPAR; ++s)
#pragma unroll
        for (int p = 0; p < NP; ++p)
#pragma unroll
            for (int mt = 0; mt < G::MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < G::NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[s][p][mt][nt][e] = 0.f;
    auto take = [](float x0, float x1, uint32_t &hi, uint32_t &lo, bool exact) {
        if (exact) hi = pack_bf16(x0, x1);
        else split_bf16x2(x0, x1, hi, lo);
    };
    // a k-pair of an operand: one float2 from the accessor (APAIR / BPAIR:
    // it returns (x(k), x(k + 1)) for even k, one 8-byte load) or two values
    auto a2 = [&](int m, int k) {
        if constexpr (APAIR) return a(m, k);
        else return make_float2(a(m, k), a(m, k + 1));
    };
    auto b2 = [&](int k, int n) {
        if constexpr (BPAIR) return b(k, n);
        else return make_float2(b(k, n), b(k + 1, n));
    };
    auto kstep = [&](int k0, float (&ac)[NP][G::MT][G::NT][4]) {
        uint32_t ah[G::MT][4], al[G::MT][4], bh[G::NT][2], bl[G::NT][2];
        const int ka = k0 + 2 * tig;
#pragma unroll
        for (int mt = 0; mt < G::MT; ++mt) {
            const int m = m0 + mt * 16 + gid;
            float2 x;
            x = a2(m, ka);         take(x.x, x.y, ah[mt][0], al[mt][0], AEX);
            x = a2(m + 8, ka);     take(x.x, x.y, ah[mt][1], al[mt][1], AEX);
            x = a2(m, ka + 8);     take(x.x, x.y, ah[mt][2], al[mt][2], AEX);
            x = a2(m + 8, ka + 8); take(x.x, x.y, ah[mt][3], al[mt][3], AEX);
        }
#pragma unroll
        for (int nt = 0; nt < G::NT; ++nt) {
            const int n = n0 + nt * 8 + gid;
            float2 y;
            y = b2(ka, n);     take(y.x, y.y, bh[nt][0], bl[nt][0], BEX);
            y = b2(ka + 8, n); take(y.x, y.y, bh[nt][1], bl[nt][1], BEX);
        }
#pragma unroll
        for (int mt = 0; mt < G::MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < G::NT; ++nt) {
                if (!AEX) mma_bf16(ac[NP - 1][mt][nt], al[mt], bh[nt]);
                if (!BEX) mma_bf16(ac[NP > 1 ? 1 : 0][mt][nt], ah[mt], bl[nt]);
                mma_bf16(ac[0][mt][nt], ah[mt], bh[nt]);
            }
    };
#pragma unroll 2
    for (int k0 = 0; k0 < K; k0 += 16 * KPAR) {
        kstep(k0, acc[0]);
        if (KPAR > 1) kstep(k0 + 16, acc[KPAR - 1]);
    }
    auto total = [&](int mt, int nt, int e) {
        float x = acc[0][0][mt][nt][e], corr = 0.f;
#pragma unroll
        for (int s = 0; s < KPAR; ++s)
#pragma unroll
            for (int p = 0; p < NP; ++p)
                if (s + p > 0) {
                    if (p > 0) corr += acc[s][p][mt][nt][e];
                    else x += acc[s][p][mt][nt][e];
                }
        return x + corr;
    };
#pragma unroll
    for (int mt = 0; mt < G::MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < G::NT; ++nt) {
            if constexpr (PAIRS) {
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    epi(mt * 2 + h, m0 + mt * 16 + gid + 8 * h, n0 + nt * 8 + 2 * tig,
                        total(mt, nt, 2 * h), total(mt, nt, 2 * h + 1));
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    epi(mt * 2 + (e >> 1), nt * 2 + (e & 1), m0 + mt * 16 + gid + 8 * (e >> 1),
                        n0 + nt * 8 + 2 * tig + (e & 1), total(mt, nt, e));
            }
        }
}

template <int M, int N, int NTH, bool AEX = false, bool BEX = false, class AF, class BF, class EPI>
__device__ __forceinline__ void bgemm(int K, AF a, BF b, EPI epi) {
    bgemm_rc<M, N, NTH, AEX, BEX>(K, a, b, [&](int, int, int m, int n, float v) { epi(m, n, v); });
}

// bgemm storing out(m, n) row-major with ld floats: two results per 8-byte store.
template <int M, int N, int NTH, bool AEX = false, bool BEX = false, class AF, class BF>
__device__ __forceinline__ void bgemm_store(int K, AF a, BF b, float *out, int ld) {
    bgemm_rc<M, N, NTH, AEX, BEX, true>(K, a, b, [&](int, int m, int n, float x0, float x1) {
        *reinterpret_cast<float2 *>(out + (size_t)m * ld + n) = make_float2(x0, x1);
    });
}

// Row of slot r and column of slot c of the calling thread in a <M, N, NTH>
// product.
template <int M, int N, int NTH>
__device__ __forceinline__ int tslot_row(int r) {
    using G = WarpGrid<M, N, NTH / 32>;
    const int warp = (threadIdx.x & (NTH - 1)) >> 5, gid = (threadIdx.x & 31) >> 2;
    return (warp / G::GN) * G::WM + (r >> 1) * 16 + gid + 8 * (r & 1);
}
template <int M, int N, int NTH>
__device__ __forceinline__ int tslot_col(int c) {
    using G = WarpGrid<M, N, NTH / 32>;
    const int warp = (threadIdx.x & (NTH - 1)) >> 5, tig = threadIdx.x & 3;
    return (warp % G::GN) * G::WN + (c >> 1) * 8 + 2 * tig + (c & 1);
}

// base[n] = first global chunk of sequence n (exclusive prefix sum of the
// sequences' chunk counts); base[num_seqs] = all chunks.
__global__ void __launch_bounds__(1024)
bwd_chunk_base_kernel(const int32_t *__restrict__ cu, int num_seqs, int total_T, int32_t *base) {
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
        int x = v;
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
            wsum[lane] = w;
        }
        __syncthreads();
        const int incl = x + (warp > 0 ? wsum[warp - 1] : 0) + carry;
        if (n < num_seqs) base[n] = incl - v;
        __syncthreads();
        if (tid == 1023) carry = incl;
        __syncthreads();
    }
    if (tid == 0) base[num_seqs] = carry;
}

// (sequence, local chunk) of global chunk gc: base[n] <= gc < base[n + 1].
__device__ __forceinline__ bool chunk_of(const int32_t *base, int num_seqs, int gc, int &n, int &c) {
    if (gc >= base[num_seqs]) return false;
    int lo = 0, hi = num_seqs;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (base[mid] <= gc) lo = mid;
        else hi = mid;
    }
    n = lo;
    c = gc - base[n];
    return true;
}

__device__ __forceinline__ void cp16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// The chunk's 64 rows of a [T, heads, 128] input (0 past the sequence's end)
// into padded fp32 rows by 16-byte asynchronous copies: fp32 rows straight
// into place; bf16 rows into the second half of the destination (rows
// 32 .. 63 of it are not yet written), converted by finish_io_rows.
template <int NT, typename IoT>
__device__ __forceinline__ void stage_io_rows(float *dst, const IoT *src, int tok0, int cl, int heads,
                                              int head) {
    const int t = threadIdx.x & (NT - 1);
    if constexpr (std::is_same<IoT, float>::value) {
        for (int e = t; e < C * D / 4; e += NT) {
            const int i = e >> 5, q = e & 31;
            float *o = dst + i * LW + 4 * q;
            if (i < cl) cp16(o, src + ((size_t)(tok0 + i) * heads + head) * D + 4 * q);
            else *reinterpret_cast<float4 *>(o) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    } else {
        char *raw = reinterpret_cast<char *>(dst + C * LW / 2);
        for (int e = t; e < C * D / 8; e += NT) {
            const int i = e >> 4, q = e & 15;
            if (i < cl) cp16(raw + i * 256 + q * 16, src + ((size_t)(tok0 + i) * heads + head) * D + 8 * q);
        }
    }
}
// The bf16 rows staged in NW destinations, converted in place: every thread
// reads its raw pieces, the block synchronises, then writes the fp32 rows.
// Called by every thread after the copies are waited for and synchronised;
// ends synchronised.
template <int NT, typename IoT, int NW>
__device__ __forceinline__ void finish_io_rows(float *const (&dst)[NW], int cl) {
    if constexpr (!std::is_same<IoT, float>::value) {
        constexpr int PER = C * D / 8 / NT;
        uint4 raw[NW][PER];
        const int t = threadIdx.x & (NT - 1);
#pragma unroll
        for (int w = 0; w < NW; ++w)
#pragma unroll
            for (int p = 0; p < PER; ++p) {
                const int e = t + p * NT, i = e >> 4, q = e & 15;
                raw[w][p] = i < cl ? *reinterpret_cast<const uint4 *>(
                                         reinterpret_cast<const char *>(dst[w] + C * LW / 2) + i * 256 + q * 16)
                                   : make_uint4(0u, 0u, 0u, 0u);
            }
        __syncthreads();
#pragma unroll
        for (int w = 0; w < NW; ++w)
#pragma unroll
            for (int p = 0; p < PER; ++p) {
                const int e = t + p * NT, i = e >> 4, q = e & 15;
                float f[8];
                bf16x8_to_f32(raw[w][p], f);
                float4 *o = reinterpret_cast<float4 *>(dst[w] + i * LW + 8 * q);
                o[0] = make_float4(f[0], f[1], f[2], f[3]);
                o[1] = make_float4(f[4], f[5], f[6], f[7]);
            }
    }
    __syncthreads();
}

// ---------------------------------------------------------------- prep ----
// One CTA per (global chunk, value head): G, beta, A (via the strictly
// lower (K K^T) o R), T = (I + A)^-1, W, U~ and P, written to the record.
constexpr int kPrepB = 256;
constexpr uint32_t PB_K = 0;                        // K [64][129] fp32 (then beta gamma K)
constexpr uint32_t PB_Q = PB_K + C * LW;            // Q [64][129]
constexpr uint32_t PB_V = PB_Q + C * LW;            // V [64][129] (then beta V)
constexpr uint32_t PB_A = PB_V + C * LW;            // A, swizzled 64 x 64 (the inverse's layout)
constexpr uint32_t PB_T = PB_A + C * C;             // T, swizzled 64 x 64
constexpr uint32_t PB_X = PB_T + C * C;             // the inverse's 1024-float scratch
constexpr uint32_t PB_TP = PB_X + 1024;             // T [64][65], zero above the diagonal
constexpr uint32_t PB_DO = PB_TP + C * LN;          // dO [64][LW]
constexpr uint32_t PB_P = PB_DO + C * LW;           // P [64][LN]
constexpr uint32_t PB_G = PB_P + C * LN;            // G [64], gamma [64], beta [64]
constexpr uint32_t PB_FLOATS = PB_G + 3 * C;
constexpr uint32_t PB_SMEM = PB_FLOATS * sizeof(float);

template <typename IoT>
__global__ void __launch_bounds__(kPrepB, 1)
bwd_prep_kernel(const IoT *__restrict__ q, const IoT *__restrict__ k, const IoT *__restrict__ v,
                const float *__restrict__ g, const float *__restrict__ beta, const IoT *__restrict__ dO,
                const int32_t *__restrict__ cu, int num_seqs, int total_T, int Hqk, int H,
                const int32_t *__restrict__ base, float *__restrict__ recs) {
    extern __shared__ __align__(16) float fs[];
    int n, c;
    const int gc = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    if (!chunk_of(base, num_seqs, gc, n, c)) return;
    int t0, len;
    sequence_range(cu, n, num_seqs, total_T, t0, len);
    const int tok0 = t0 + c * C, cl = min(C, len - c * C), hq = h / (H / Hqk);
    float *rec = recs + ((size_t)gc * H + h) * R_FLOATS;
    float *Ks = fs + PB_K, *Qs = fs + PB_Q, *Vs = fs + PB_V, *Tp = fs + PB_TP, *DOs = fs + PB_DO,
          *Ps = fs + PB_P;
    float *Gs = fs + PB_G, *gam = Gs + C, *Bs = gam + C;
    // the chunk's rows of k, q, v and dO, every copy in flight at once
    stage_io_rows<kPrepB>(Ks, k, tok0, cl, Hqk, hq);
    stage_io_rows<kPrepB>(Qs, q, tok0, cl, Hqk, hq);
    stage_io_rows<kPrepB>(Vs, v, tok0, cl, H, h);
    stage_io_rows<kPrepB>(DOs, dO, tok0, cl, H, h);
    cp_commit();
    if (tid < 32) {   // gates of tokens 2 tid, 2 tid + 1: clamped, cumulated, 0 past the end
        const int i0 = 2 * tid, i1 = i0 + 1;
        const float g0 = i0 < cl ? clamp_log_gate(g[(size_t)(tok0 + i0) * H + h]) : 0.f;
        const float g1 = i1 < cl ? clamp_log_gate(g[(size_t)(tok0 + i1) * H + h]) : 0.f;
        float incl = g0 + g1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, incl, off);
            if (tid >= off) incl += y;
        }
        Gs[i0] = incl - g1;
        Gs[i1] = incl;
        gam[i0] = __expf(incl - g1);
        gam[i1] = __expf(incl);
        Bs[i0] = i0 < cl ? beta[(size_t)(tok0 + i0) * H + h] : 0.f;
        Bs[i1] = i1 < cl ? beta[(size_t)(tok0 + i1) * H + h] : 0.f;
    }
    cp_wait<0>();
    __syncthreads();
    {
        float *const rows[4] = {Ks, Qs, Vs, DOs};
        finish_io_rows<kPrepB, IoT>(rows, cl);   // ends synchronised
    }
    // (K K^T) o R (strictly lower) -> record and A = diag(beta) of it; P -> record
    float *Af = fs + PB_A;
    constexpr bool kX = kIoExact<IoT>;
    tgemm<C, C, kPrepB, kX, kX>(D, [&](int i, int d) { return Ks[i * LW + d]; },
                       [&](int d, int j) { return Ks[j * LW + d]; },
                       [&](int i, int j, float x) {
                           const float ar = j < i ? x * __expf(Gs[i] - Gs[j]) : 0.f;
                           rec[R_AR + i * C + j] = ar;
                           Af[ax(i, j)] = Bs[i] * ar;
                       });
    tgemm<C, C, kPrepB, kX, kX>(D, [&](int i, int d) { return Qs[i * LW + d]; },
                       [&](int d, int j) { return Ks[j * LW + d]; },
                       [&](int i, int j, float x) {
                           const float pv = j <= i ? x * __expf(Gs[i] - Gs[j]) : 0.f;
                           rec[R_P + j * C + i] = pv;
                           Ps[i * LN + j] = pv;
                       });
    __syncthreads();
    unit_lower_inverse_f32(Af, fs + PB_T, fs + PB_X, tid);   // ends synchronised
    for (int e = tid; e < C * C; e += kPrepB) {
        const int i = e >> 6, j = e & 63;
        const float t = j <= i ? (fs + PB_T)[ax(i, j)] : 0.f;
        Tp[i * LN + j] = t;
        rec[R_T + e] = t;
    }
    // K^ and diag(gamma) Q to the record
    const float GCp = Gs[C - 1];
    for (int e = tid; e < C * D; e += kPrepB) {
        const int i = e >> 7, d = e & 127;
        rec[R_KH + e] = Ks[i * LW + d] * __expf(GCp - Gs[i]);
        rec[R_QT + e] = Qs[i * LW + d] * gam[i];
    }
    if (tid < C) {
        rec[R_G + tid] = Gs[tid];
        rec[R_B + tid] = Bs[tid];
    }
    __syncthreads();
    // W = T diag(beta gamma) K and U~ = T diag(beta) V, the scales taken
    // with T so that K and V stay exact operands
    bgemm_store<C, D, kPrepB, false, kX>(C, [&](int i, int j) { return Tp[i * LN + j] * Bs[j] * gam[j]; },
                                          [&](int j, int d) { return Ks[j * LW + d]; }, rec + R_W, D);
    bgemm_store<C, D, kPrepB, false, kX>(C, [&](int i, int j) { return Tp[i * LN + j] * Bs[j]; },
                                          [&](int j, int d) { return Vs[j * LW + d]; }, rec + R_UT, D);
    // the upstream gradient's terms of the adjoint chain, which depend on the
    // chunk alone: Y = dO^T diag(gamma) Q and Z = P^T dO
    bgemm_store<D, D, kPrepB, kX>(C, [&](int r, int i) { return DOs[i * LW + r]; },
                                   [&](int i, int d) { return Qs[i * LW + d] * gam[i]; }, rec + R_Y, D);
    bgemm_store<C, D, kPrepB, false, kX>(C, [&](int j, int i) { return Ps[i * LN + j]; },
                                          [&](int i, int r) { return DOs[i * LW + r]; }, rec + R_Z, D);
}

// ------------------------------------------------------ forward / reverse ----
// 256 threads per (sequence, value head, block of 16 state rows) and chain
// (the forward chain of the state, the reverse chain of its adjoint; one CTA
// of 512 threads holds both, see bwd_chains_kernel).  The rows of the state
// and of its adjoint are independent, so the row blocks share nothing.
// Each chunk takes two products over operands staged in shared memory by
// 16-byte asynchronous copies.  An operand is reloaded for the next chunk as
// soon as its product is done, so that its copy runs during the other
// product.  Rows read in k-pairs (8-byte loads) are padded to 8 mod 32
// floats, rows read down a column to 4 mod 32: both without bank conflicts.
constexpr int kChainThreads = 256;
constexpr int LW4 = D + 4;   // rows of a K x N B operand (read down a column)
constexpr int LW8 = D + 8;   // rows read in k-pairs by 8-byte loads
constexpr int LN8 = C + 8;
static_assert(kChainThreads == C * 4, "one 16-byte piece of a column strip per thread");

// 64 x 128 floats of a record field into rows of ld floats.
__device__ __forceinline__ void stage_c_by_d(float *dst, int ld, const float *src) {
#pragma unroll 8
    for (int e = threadIdx.x & (kChainThreads - 1); e < C * D / 4; e += kChainThreads)
        cp16(dst + (e >> 5) * ld + (e & 31) * 4, src + e * 4);
}
// rows x cols fp32 (cols a multiple of 4) from the record into rows of ld
// floats (16-byte aligned), by 16-byte asynchronous copies over NT threads.
template <int NT>
__device__ __forceinline__ void copy_rows_async(float *dst, int ld, const float *src, int rows, int cols) {
    const int q4 = cols / 4, total = rows * q4;
    for (int e = threadIdx.x & (NT - 1); e < total; e += NT)
        cp16(dst + (e / q4) * ld + (e % q4) * 4, src + e * 4);
}

// Columns r0 .. r0 + 15 of a 64 x 128 record field into rows of 16 floats.
__device__ __forceinline__ void stage_strip(float *dst, const float *src, int r0) {
    const int e = threadIdx.x & (kChainThreads - 1);
    cp16(dst + (e >> 2) * kRowBlock + (e & 3) * 4, src + (e >> 2) * D + r0 + (e & 3) * 4);
}
// The chunk's 64 floats of G.
__device__ __forceinline__ void stage_g(float *dst, const float *src) {
    const int e = threadIdx.x & (kChainThreads - 1);
    if (e < C / 4) cp16(dst + e * 4, src + e * 4);
}

__device__ __forceinline__ float4 lds4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
// The CTA's 16 rows (rows of ld floats) -> rows r0 .. r0 + 15 of a [128][128] field.
__device__ __forceinline__ void store_rows(float *dst, const float *rows, int ld, int r0) {
#pragma unroll
    for (int e = threadIdx.x & (kChainThreads - 1); e < kRowBlock * D / 4; e += kChainThreads) {
        const int r = e >> 5, q = e & 31;
        *reinterpret_cast<float4 *>(dst + (size_t)(r0 + r) * D + 4 * q) = lds4(rows + r * ld + 4 * q);
    }
}

constexpr uint32_t CF_S = 0;                             // S rows [16][LW8]
constexpr uint32_t CF_UT = CF_S + kRowBlock * LW8;       // U^T [16][LN8]
constexpr uint32_t CF_W = CF_UT + kRowBlock * LN8;       // W [64][LW8]
constexpr uint32_t CF_KH = CF_W + C * LW8;               // K^ [64][LW4]
constexpr uint32_t CF_US = CF_KH + C * LW4;              // U~ columns r0 .. r0 + 15 [64][16]
constexpr uint32_t CF_G = CF_US + C * kRowBlock;         // G [64]
constexpr uint32_t CF_SMEM = (CF_G + C) * sizeof(float);

__device__ __forceinline__ void forward_chain(float *fs, const float *__restrict__ h0, const int32_t *__restrict__ cu, int num_seqs,
                   int total_T, int H, const int32_t *__restrict__ base, long long slots,
                   float *__restrict__ recs) {
    const int chain = blockIdx.x, h = chain % H, n = chain / H, r0 = blockIdx.y * kRowBlock;
    const int tid = threadIdx.x & (kChainThreads - 1);
    int t0, len;
    sequence_range(cu, n, num_seqs, total_T, t0, len);
    const int b0 = base[n];
    // a malformed cu_seqlens can claim more chunks than the records hold
    const int nch = (int)min((long long)(len + C - 1) / C, max(slots - b0, 0ll));
    float *Sr = fs + CF_S, *Ut = fs + CF_UT, *Ws = fs + CF_W, *Kh = fs + CF_KH, *Us = fs + CF_US,
          *Gs = fs + CF_G;
    auto rec_of = [&](int c) { return recs + ((size_t)(b0 + c) * H + h) * R_FLOATS; };
    for (int e = tid; e < kRowBlock * D; e += kChainThreads) {
        const int r = e >> 7, d = e & 127;
        Sr[r * LW8 + d] = h0 != nullptr ? h0[((size_t)chain * D + r0 + r) * D + d] : 0.f;
    }
    // copy groups, in order: {W, U~} and {K^, G} of every chunk
    if (nch > 0) {
        stage_c_by_d(Ws, LW8, rec_of(0) + R_W);
        stage_strip(Us, rec_of(0) + R_UT, r0);
        cp_commit();
        stage_c_by_d(Kh, LW4, rec_of(0) + R_KH);
        stage_g(Gs, rec_of(0) + R_G);
        cp_commit();
    }
    for (int c = 0; c < nch; ++c) {
        float *rec = rec_of(c);
        cp_wait<1>();
        group_sync(1);   // W, U~ of chunk c and the state rows in place
        if (tid == 0 && blockIdx.y == 0 && c + 2 < nch) {   // chunk c + 2 towards L2
            const float *nx = rec_of(c + 2);
            tc::bulk_prefetch_l2(nx + R_W, 2 * C * D * sizeof(float));   // W and U~
            tc::bulk_prefetch_l2(nx + R_KH, C * D * sizeof(float));
            tc::bulk_prefetch_l2(nx + R_G, C * sizeof(float));
        }
        store_rows(rec + R_S, Sr, LW8, r0);
        // U[j][r0 + r] = U~[j][r0 + r] - sum_d W[j][d] S[r][d]
        bgemm_rc<C, kRowBlock, kChainThreads, false, false, true, 2, true, true, true>(
            D, [&](int j, int d) { return *reinterpret_cast<const float2 *>(Ws + j * LW8 + d); },
            [&](int d, int r) { return *reinterpret_cast<const float2 *>(Sr + r * LW8 + d); },
            [&](int, int j, int r, float x0, float x1) {
                const float u0 = Us[j * kRowBlock + r] - x0, u1 = Us[j * kRowBlock + r + 1] - x1;
                Ut[r * LN8 + j] = u0;
                Ut[(r + 1) * LN8 + j] = u1;
                *reinterpret_cast<float2 *>(rec + R_U + j * D + r0 + r) = make_float2(u0, u1);
            });
        group_sync(1);   // W and U~ consumed, U^T complete
        if (c + 1 < nch) {
            stage_c_by_d(Ws, LW8, rec_of(c + 1) + R_W);
            stage_strip(Us, rec_of(c + 1) + R_UT, r0);
        }
        cp_commit();
        cp_wait<1>();
        group_sync(1);   // K^ and G of chunk c in place
        {   // S[r][d] = e^{G_C} S[r][d] + sum_j U[j][r] K^[j][d]
            const float gC = __expf(Gs[C - 1]);
            bgemm_rc<kRowBlock, D, kChainThreads, false, false, true, 2, true, true, false>(
                C, [&](int r, int j) { return *reinterpret_cast<const float2 *>(Ut + r * LN8 + j); },
                [&](int j, int d) { return Kh[j * LW4 + d]; },
                                               [&](int, int r, int d, float x0, float x1) {
                                                   float2 *p = reinterpret_cast<float2 *>(Sr + r * LW8 + d);
                                                   const float2 s = *p;
                                                   *p = make_float2(fmaf(gC, s.x, x0), fmaf(gC, s.y, x1));
                                               });
        }
        group_sync(1);   // K^ and G consumed
        if (c + 1 < nch) {
            stage_c_by_d(Kh, LW4, rec_of(c + 1) + R_KH);
            stage_g(Gs, rec_of(c + 1) + R_G);
        }
        cp_commit();
    }
    cp_wait<0>();
}

constexpr uint32_t CR_L = 0;                             // L rows [16][LW8]
constexpr uint32_t CR_DUT = CR_L + kRowBlock * LW8;      // dU^T [16][LN8]
constexpr uint32_t CR_KH = CR_DUT + kRowBlock * LN8;     // K^ [64][LW8]
constexpr uint32_t CR_ZS = CR_KH + C * LW8;              // Z columns r0 .. r0 + 15 [64][16]
constexpr uint32_t CR_W = CR_ZS + C * kRowBlock;         // W [64][LW4]
constexpr uint32_t CR_YS = CR_W + C * LW4;               // Y rows r0 .. r0 + 15 [16][LW4]
constexpr uint32_t CR_G = CR_YS + kRowBlock * LW4;       // G [64]
constexpr uint32_t CR_SMEM = (CR_G + C) * sizeof(float);

// Rows r0 .. r0 + 15 of a [128][128] record field into rows of LW4 floats.
__device__ __forceinline__ void stage_row_block(float *dst, const float *src, int r0) {
#pragma unroll
    for (int e = threadIdx.x & (kChainThreads - 1); e < kRowBlock * D / 4; e += kChainThreads)
        cp16(dst + (e >> 5) * LW4 + (e & 31) * 4, src + (size_t)r0 * D + e * 4);
}

// The adjoint chain, chunks last to first: with the chunk's upstream terms
// Y = dO^T diag(gamma) Q and Z = P^T dO taken from the record,
//   dU = Z + K^ L'^T,   L = e^{G_C} L' + Y - dU^T W
// (L' the adjoint of the state leaving the chunk, L of the one entering it).
__device__ __forceinline__ void reverse_chain(float *fs, const float *__restrict__ dSf, float *__restrict__ dh0,
                   const int32_t *__restrict__ cu, int num_seqs, int total_T, int H,
                   const int32_t *__restrict__ base, long long slots, float *__restrict__ recs) {
    const int chain = blockIdx.x, h = chain % H, n = chain / H, r0 = blockIdx.y * kRowBlock;
    const int tid = threadIdx.x & (kChainThreads - 1);
    int t0, len;
    sequence_range(cu, n, num_seqs, total_T, t0, len);
    const int b0 = base[n];
    const int nch = (int)min((long long)(len + C - 1) / C, max(slots - b0, 0ll));
    float *Lr = fs + CR_L, *dUt = fs + CR_DUT, *Kh = fs + CR_KH, *Zs = fs + CR_ZS, *Ws = fs + CR_W,
          *Ys = fs + CR_YS, *Gs = fs + CR_G;
    auto rec_of = [&](int c) { return recs + ((size_t)(b0 + c) * H + h) * R_FLOATS; };
    for (int e = tid; e < kRowBlock * D; e += kChainThreads) {
        const int r = e >> 7, d = e & 127;
        Lr[r * LW8 + d] = dSf != nullptr ? dSf[((size_t)chain * D + r0 + r) * D + d] : 0.f;
    }
    // copy groups, in order: {K^, Z} and {W, Y, G} of every chunk
    if (nch > 0) {
        stage_c_by_d(Kh, LW8, rec_of(nch - 1) + R_KH);
        stage_strip(Zs, rec_of(nch - 1) + R_Z, r0);
        cp_commit();
        stage_c_by_d(Ws, LW4, rec_of(nch - 1) + R_W);
        stage_row_block(Ys, rec_of(nch - 1) + R_Y, r0);
        stage_g(Gs, rec_of(nch - 1) + R_G);
        cp_commit();
    }
    for (int c = nch - 1; c >= 0; --c) {
        float *rec = rec_of(c);
        cp_wait<1>();
        group_sync(2);   // K^ and Z of chunk c and the adjoint rows in place
        if (tid == 0 && blockIdx.y == 0 && c >= 2) {   // chunk c - 2 towards L2
            const float *pv = rec_of(c - 2);
            tc::bulk_prefetch_l2(pv + R_KH, C * D * sizeof(float));
            tc::bulk_prefetch_l2(pv + R_W, C * D * sizeof(float));
            tc::bulk_prefetch_l2(pv + R_Y, D * D * sizeof(float));
            tc::bulk_prefetch_l2(pv + R_Z, C * D * sizeof(float));
            tc::bulk_prefetch_l2(pv + R_G, C * sizeof(float));
        }
        store_rows(rec + R_L, Lr, LW8, r0);
        // dU[j][r0 + r] = Z[j][r0 + r] + sum_d K^[j][d] L[r][d]
        bgemm_rc<C, kRowBlock, kChainThreads, false, false, true, 2, true, true, true>(
            D, [&](int j, int d) { return *reinterpret_cast<const float2 *>(Kh + j * LW8 + d); },
            [&](int d, int r) { return *reinterpret_cast<const float2 *>(Lr + r * LW8 + d); },
            [&](int, int j, int r, float x0, float x1) {
                const float v0 = Zs[j * kRowBlock + r] + x0, v1 = Zs[j * kRowBlock + r + 1] + x1;
                dUt[r * LN8 + j] = v0;
                dUt[(r + 1) * LN8 + j] = v1;
                *reinterpret_cast<float2 *>(rec + R_DU + j * D + r0 + r) = make_float2(v0, v1);
            });
        group_sync(2);   // K^ and Z consumed, dU^T complete
        if (c > 0) {
            stage_c_by_d(Kh, LW8, rec_of(c - 1) + R_KH);
            stage_strip(Zs, rec_of(c - 1) + R_Z, r0);
        }
        cp_commit();
        cp_wait<1>();
        group_sync(2);   // W, Y and G of chunk c in place
        {   // L[r][d] = e^{G_C} L[r][d] + Y[r0 + r][d] - sum_j dU[j][r] W[j][d]
            const float gC = __expf(Gs[C - 1]);
            bgemm_rc<kRowBlock, D, kChainThreads, false, false, true, 2, true, true, false>(
                C, [&](int r, int j) { return *reinterpret_cast<const float2 *>(dUt + r * LN8 + j); },
                [&](int j, int d) { return Ws[j * LW4 + d]; },
                [&](int, int r, int d, float x0, float x1) {
                    float2 *p = reinterpret_cast<float2 *>(Lr + r * LW8 + d);
                    const float2 l = *p, y = *reinterpret_cast<const float2 *>(Ys + r * LW4 + d);
                    *p = make_float2(fmaf(gC, l.x, y.x - x0), fmaf(gC, l.y, y.y - x1));
                });
        }
        group_sync(2);   // W, Y and G consumed
        if (c > 0) {
            stage_c_by_d(Ws, LW4, rec_of(c - 1) + R_W);
            stage_row_block(Ys, rec_of(c - 1) + R_Y, r0);
            stage_g(Gs, rec_of(c - 1) + R_G);
        }
        cp_commit();
    }
    cp_wait<0>();
    group_sync(2);
    if (dh0 != nullptr) {
        for (int e = tid; e < kRowBlock * D; e += kChainThreads) {
            const int r = e >> 7, d = e & 127;
            dh0[((size_t)chain * D + r0 + r) * D + d] = Lr[r * LW8 + d];
        }
    }
}

// Both chains in one CTA of 512 threads per (sequence, head, 16 rows):
// warps 0-7 carry the state forward, warps 8-15 the adjoint backward, each
// half on its own named barrier.  The two share nothing (the chunk-local
// gradients need both, afterwards), so the SM's tensor pipe serves both.
constexpr uint32_t CH_SMEM = CF_SMEM + CR_SMEM;
__global__ void __launch_bounds__(2 * kChainThreads, 1)
bwd_chains_kernel(const float *__restrict__ h0, const float *__restrict__ dSf,
                  float *__restrict__ dh0, const int32_t *__restrict__ cu, int num_seqs,
                  int total_T, int H, const int32_t *__restrict__ base, long long slots,
                  float *__restrict__ recs) {
    extern __shared__ __align__(16) float fs[];
    if (threadIdx.x < kChainThreads)
        forward_chain(fs, h0, cu, num_seqs, total_T, H, base, slots, recs);
    else
        reverse_chain(fs + CF_SMEM / sizeof(float), dSf, dh0, cu, num_seqs, total_T, H, base, slots, recs);
}

// --------------------------------------------------------------- local ----
// One CTA per (global chunk, value head): every gradient of the chunk's
// tokens.  Shared memory (floats, rows of LW = 132 or LN = 68) is reused
// phase by phase:
//   RA [128][LW]: L', then S, then U [64][LW], then K [64][LW]
//   RB [64][LW]:  U, then dU, then Y = dT T^T and dA o A / beta ([64][LN]), then Q
//   RC [64][LW]:  K^, then dW, then (K K^T) o R and dA o A + dP o P ([64][LN])
//   RD [64][LW]:  dO, then V (RD .. N3 hold S, dense, during phase A)
//   N1, N2, N3 [64][LN]: T then P^T; dP then its product form; dT then dA
// and the per-token adjoints dG, dbeta (shared atomics).
constexpr uint32_t LB_RA = 0;
constexpr uint32_t LB_RB = LB_RA + D * LW;
constexpr uint32_t LB_RC = LB_RB + C * LW;
constexpr uint32_t LB_RD = LB_RC + C * LW;
constexpr uint32_t LB_N1 = LB_RD + C * LW;
constexpr uint32_t LB_N2 = LB_N1 + C * LN;
constexpr uint32_t LB_N3 = LB_N2 + C * LN;
constexpr uint32_t LB_G = LB_N3 + C * LN;     // G, gamma, beta, dG, dbeta [64] each
constexpr uint32_t LB_MISC = LB_G + 5 * C;    // dG_C, <S, L'>
constexpr uint32_t LB_FLOATS = LB_MISC + 8;
constexpr uint32_t LB_SMEM = LB_FLOATS * sizeof(float);

template <typename IoT>
__global__ void __launch_bounds__(kLocalThreads, 1)
bwd_local_kernel(const IoT *__restrict__ q, const IoT *__restrict__ k, const IoT *__restrict__ v,
                 const float *__restrict__ g, const IoT *__restrict__ dO,
                 const int32_t *__restrict__ cu, int num_seqs, int total_T, int Hqk, int H,
                 const int32_t *__restrict__ base, const float *__restrict__ recs,
                 float *__restrict__ dq, float *__restrict__ dk, float *__restrict__ dv,
                 float *__restrict__ dg, float *__restrict__ dbeta) {
    extern __shared__ __align__(16) float fs[];
    int n, c;
    const int gc = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    if (!chunk_of(base, num_seqs, gc, n, c)) return;
    int t0, len;
    sequence_range(cu, n, num_seqs, total_T, t0, len);
    const int tok0 = t0 + c * C, cl = min(C, len - c * C), hq = h / (H / Hqk);
    const float *rec = recs + ((size_t)gc * H + h) * R_FLOATS;
    float *RA = fs + LB_RA, *RB = fs + LB_RB, *RC = fs + LB_RC, *RD = fs + LB_RD;
    float *N1 = fs + LB_N1, *N2 = fs + LB_N2, *N3 = fs + LB_N3;
    float *Gs = fs + LB_G, *gam = Gs + C, *Bs = gam + C, *dG = Bs + C, *dB = dG + C;
    float *misc = fs + LB_MISC;
    auto qk_at = [&](float *base_, int i, int d) { return base_ + ((size_t)(tok0 + i) * Hqk + hq) * D + d; };
    static_assert(2 * WarpGrid<C, D, kLocalThreads / 32>::MT == kLocTM &&
                      2 * WarpGrid<C, D, kLocalThreads / 32>::NT == kLocTN,
                  "slots of a <C, D> product");
    // dk and dq of the chunk's rows, summed over the product terms in the
    // registers of the <C, D> product slots
    float dkacc[kLocTM][kLocTN], dqacc[kLocTM][kLocTN];
    // per-row sums over the slots of a <C, D> product -> dst[row] (shared)
    auto flush_rows = [&](float *dst, const float (&acc)[kLocTM]) {
#pragma unroll
        for (int r = 0; r < kLocTM; ++r) {
            float x = acc[r];
            x += __shfl_xor_sync(0xffffffffu, x, 1);
            x += __shfl_xor_sync(0xffffffffu, x, 2);
            if ((tid & 3) == 0) atomicAdd(&dst[tslot_row<C, D, kLocalThreads>(r)], x);
        }
    };
    // everything the later phases read towards L2 while phase A runs: the
    // record's P, T, (K K^T) o R, G, beta and U .. gamma Q (64 KiB pieces),
    // and the chunk's rows of q, k, v and dO
    if (tid == 0) {
        tc::bulk_prefetch_l2(rec + R_P, (3 * C * C + 2 * C) * sizeof(float));
        for (size_t o = R_U; o < R_Y; o += 16384)
            tc::bulk_prefetch_l2(rec + o, (uint32_t)(min((size_t)16384, R_Y - o) * sizeof(float)));
    }
    static_assert(kLocalThreads == 4 * C, "one input row per thread");
    {
        const int w = tid / C, i = tid % C;   // one row of q, k, v or dO per thread
        if (i < cl) {
            const IoT *src = w == 0 ? q + ((size_t)(tok0 + i) * Hqk + hq) * D
                           : w == 1 ? k + ((size_t)(tok0 + i) * Hqk + hq) * D
                           : w == 2 ? v + ((size_t)(tok0 + i) * H + h) * D
                                    : dO + ((size_t)(tok0 + i) * H + h) * D;
            tc::bulk_prefetch_l2(src, D * sizeof(IoT));
        }
    }

    // ---- phase A: dK^ = U L' and <S, L'> --------------------------------------
    copy_rows_async<kLocalThreads>(RA, LW, rec + R_L, D, D);
    copy_rows_async<kLocalThreads>(RB, LW, rec + R_U, C, D);
    copy_rows_async<kLocalThreads>(RC, LW, rec + R_KH, C, D);
    float *Sd = RD;   // S, dense 128 x 128, in the buffers phase A leaves free (RD .. N3)
    static_assert(LB_G - LB_RD >= D * D, "room for S");
    copy_rows_async<kLocalThreads>(Sd, D, rec + R_S, D, D);
    cp_commit();
    if (tid < C) {
        Gs[tid] = rec[R_G + tid];
        gam[tid] = __expf(rec[R_G + tid]);
        Bs[tid] = rec[R_B + tid];
        dG[tid] = 0.f;
        dB[tid] = 0.f;
    }
    if (tid < 8) misc[tid] = 0.f;
    cp_wait<0>();
    __syncthreads();
    const float GC = Gs[C - 1], gC = __expf(GC);
    {
        float part = 0.f;   // <S, L'> over this thread's entries
#pragma unroll 8
        for (int e = tid; e < D * D / 4; e += kLocalThreads) {
            const float4 x = *reinterpret_cast<const float4 *>(Sd + e * 4);
            const float4 y = *reinterpret_cast<const float4 *>(RA + (e >> 5) * LW + (e & 31) * 4);
            part = fmaf(x.x, y.x, fmaf(x.y, y.y, fmaf(x.z, y.z, fmaf(x.w, y.w, part))));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        if ((tid & 31) == 0) atomicAdd(&misc[1], part);
    }
    __syncthreads();
    {
        float rowacc[4] = {0.f, 0.f, 0.f, 0.f}, gcacc = 0.f;
        bgemm_rc<C, D, kLocalThreads>(D, [&](int j, int r) { return RB[j * LW + r]; },
                                  [&](int r, int d) { return RA[r * LW + d]; },
                                  [&](int tr, int tc, int j, int d, float x) {
                                      dkacc[tr][tc] = __expf(GC - Gs[j]) * x;
                                      const float t = RC[j * LW + d] * x;
                                      rowacc[tr] -= t;
                                      gcacc += t;
                                  });
        flush_rows(dG, rowacc);
        atomicAdd(&misc[0], gcacc);
    }
    __syncthreads();

    // ---- phase B: dW = -dU S, d(gamma Q) = dO S ---------------------------------
    copy_rows_async<kLocalThreads>(RA, LW, rec + R_S, D, D);
    copy_rows_async<kLocalThreads>(RB, LW, rec + R_DU, C, D);
    stage_io_rows<kLocalThreads>(RD, dO, tok0, cl, H, h);
    cp_commit();
    cp_wait<0>();
    __syncthreads();
    {
        float *const rows[1] = {RD};
        finish_io_rows<kLocalThreads, IoT>(rows, cl);
    }
    bgemm<C, D, kLocalThreads>(D, [&](int j, int r) { return RB[j * LW + r]; },
                              [&](int r, int d) { return RA[r * LW + d]; },
                              [&](int j, int d, float x) { RC[j * LW + d] = -x; });
    {
        float rowacc[4] = {0.f, 0.f, 0.f, 0.f};
        bgemm_rc<C, D, kLocalThreads, kIoExact<IoT>>(D, [&](int i, int r) { return RD[i * LW + r]; },
                                  [&](int r, int d) { return RA[r * LW + d]; },
                                  [&](int tr, int tc, int i, int d, float x) {
                                      dqacc[tr][tc] = gam[i] * x;
                                      if (i < cl) rowacc[tr] += rec[R_QT + i * D + d] * x;
                                  });
        flush_rows(dG, rowacc);
    }
    __syncthreads();

    // ---- phase C: dP, T^T dU, T^T dW, dT ---------------------------------------
    copy_rows_async<kLocalThreads>(RA, LW, rec + R_U, C, D);
    copy_rows_async<kLocalThreads>(N1, LN, rec + R_T, C, C);
    cp_commit();
    cp_wait<0>();
    __syncthreads();
    bgemm<C, C, kLocalThreads, kIoExact<IoT>>(D, [&](int i, int r) { return RD[i * LW + r]; },
                              [&](int r, int j) { return RA[j * LW + r]; },
                              [&](int i, int j, float x) { N2[i * LN + j] = j <= i ? x : 0.f; });
    __syncthreads();
    stage_io_rows<kLocalThreads>(RD, v, tok0, cl, H, h);
    stage_io_rows<kLocalThreads>(RA, k, tok0, cl, Hqk, hq);
    cp_commit();
    cp_wait<0>();
    __syncthreads();
    {
        float *const rows[2] = {RD, RA};
        finish_io_rows<kLocalThreads, IoT>(rows, cl);
    }
    {
        float rowacc[4] = {0.f, 0.f, 0.f, 0.f};
        bgemm_rc<C, D, kLocalThreads, false, false, true>(
            C, [&](int j, int i) { return N1[i * LN + j]; }, [&](int i, int r) { return RB[i * LW + r]; },
            [&](int tr, int j, int r, float x0, float x1) {
                if (j < cl)
                    *reinterpret_cast<float2 *>(dv + ((size_t)(tok0 + j) * H + h) * D + r) =
                        make_float2(Bs[j] * x0, Bs[j] * x1);
                rowacc[tr] += RD[j * LW + r] * x0 + RD[j * LW + r + 1] * x1;
            });
        flush_rows(dB, rowacc);
    }
    {
        float bacc[4] = {0.f, 0.f, 0.f, 0.f}, gacc[4] = {0.f, 0.f, 0.f, 0.f};
        bgemm_rc<C, D, kLocalThreads>(C, [&](int j, int i) { return N1[i * LN + j]; },
                                  [&](int i, int d) { return RC[i * LW + d]; },
                                  [&](int tr, int tc, int j, int d, float x) {
                                      dkacc[tr][tc] += Bs[j] * gam[j] * x;
                                      const float t = RA[j * LW + d] * x;
                                      bacc[tr] += gam[j] * t;
                                      gacc[tr] += Bs[j] * gam[j] * t;
                                  });
        flush_rows(dB, bacc);
        flush_rows(dG, gacc);
    }
    bgemm<C, C, kLocalThreads, false, kIoExact<IoT>>(
        D, [&](int i, int r) { return RB[i * LW + r]; }, [&](int r, int j) { return RD[j * LW + r]; },
        [&](int i, int j, float x) { N3[i * LN + j] = Bs[j] * x; });
    bgemm<C, C, kLocalThreads, false, kIoExact<IoT>>(
        D, [&](int i, int d) { return RC[i * LW + d]; }, [&](int d, int j) { return RA[j * LW + d]; },
        [&](int i, int j, float x) { N3[i * LN + j] += Bs[j] * gam[j] * x; });
    __syncthreads();

    // ---- phase D: dA = -T^T dT T^T, then the A and P terms ------------------------
    float *Y = RB;   // [64][65]
    bgemm<C, C, kLocalThreads>(C, [&](int i, int m) { return N3[i * LN + m]; },
                              [&](int m, int j) { return N1[j * LN + m]; },
                              [&](int i, int j, float x) { Y[i * LN + j] = x; });
    __syncthreads();
    bgemm<C, C, kLocalThreads>(C, [&](int i, int m) { return N1[m * LN + i]; },
                              [&](int m, int j) { return Y[m * LN + j]; },
                              [&](int i, int j, float x) { N3[i * LN + j] = j < i ? -x : 0.f; });
    __syncthreads();
    float *AR = RC;   // [64][65]
    copy_rows_async<kLocalThreads>(AR, LN, rec + R_AR, C, C);
    copy_rows_async<kLocalThreads>(N1, LN, rec + R_P, C, C);
    cp_commit();
    cp_wait<0>();
    __syncthreads();
    {
        // dA o A + dP o P over AR (each element read, then written, by one
        // thread) and dA o A / beta_i over the finished Y; then their row
        // sums (dG_i, dbeta_i) and column sums (dG_j), each by one thread
        float *Es = AR, *Bq = RB;
        for (int e = tid; e < C * C; e += kLocalThreads) {
            const int i = e >> 6, j = e & 63;
            const float R = j <= i ? __expf(Gs[i] - Gs[j]) : 0.f;
            const float da = N3[i * LN + j], ar = AR[i * LN + j];
            const float dp = N2[i * LN + j], ep = dp * N1[j * LN + i];   // dP o P (N1 holds P^T)
            Es[i * LN + j] = da * Bs[i] * ar + ep;
            Bq[i * LN + j] = da * ar;
            N3[i * LN + j] = da * Bs[i] * R;             // M = dA o beta_i R
            N2[i * LN + j] = dp * R;                     // dP o R
        }
        __syncthreads();
        if (tid < C) {   // row tid, columns in a staggered order (no bank conflicts)
            float se = 0.f, sb = 0.f;
#pragma unroll 8
            for (int s_ = 0; s_ < C; ++s_) {
                const int j = (s_ + tid) & (C - 1);
                se += Es[tid * LN + j];
                sb += Bq[tid * LN + j];
            }
            atomicAdd(&dG[tid], se);
            atomicAdd(&dB[tid], sb);
        } else if (tid < 2 * C) {   // column tid - C
            const int j = tid - C;
            float se = 0.f;
#pragma unroll 8
            for (int i = 0; i < C; ++i) se += Es[i * LN + j];
            atomicAdd(&dG[j], -se);
        }
        __syncthreads();
    }
    stage_io_rows<kLocalThreads>(RB, q, tok0, cl, Hqk, hq);   // Q rows over the finished Y
    cp_commit();
    cp_wait<0>();
    __syncthreads();
    {
        float *const rows[1] = {RB};
        finish_io_rows<kLocalThreads, IoT>(rows, cl);
    }
    auto add_dk = [&](int tr, int tc, int, int, float x) { dkacc[tr][tc] += x; };
    constexpr bool kX = kIoExact<IoT>;
    // dk_i += sum_j M_ij k_j and dk_j += sum_i M_ij k_i: one product with M + M^T
    bgemm_rc<C, D, kLocalThreads, false, kX>(
        C, [&](int i, int j) { return N3[i * LN + j] + N3[j * LN + i]; },
        [&](int j, int d) { return RA[j * LW + d]; }, add_dk);
    bgemm_rc<C, D, kLocalThreads, false, kX>(C, [&](int i, int j) { return N2[i * LN + j]; },
                                                        [&](int j, int d) { return RA[j * LW + d]; },
                                                        [&](int tr, int tc, int, int, float x) { dqacc[tr][tc] += x; });
    bgemm_rc<C, D, kLocalThreads, false, kX>(C, [&](int j, int i) { return N2[i * LN + j]; },
                                                        [&](int i, int d) { return RB[i * LW + d]; }, add_dk);
    {
        // one sum per element: a store when the chunk's head owns its q/k
        // head, else an atomic (the value heads of a group share it)
        const bool sole = H == Hqk;
#pragma unroll
        for (int r = 0; r < kLocTM; ++r) {
            const int i = tslot_row<C, D, kLocalThreads>(r);
            if (i >= cl) continue;
#pragma unroll
            for (int c = 0; c < kLocTN; c += 2) {   // slots c, c + 1: columns d, d + 1
                const int d = tslot_col<C, D, kLocalThreads>(c);
                if (sole) {
                    *reinterpret_cast<float2 *>(qk_at(dk, i, d)) = make_float2(dkacc[r][c], dkacc[r][c + 1]);
                    *reinterpret_cast<float2 *>(qk_at(dq, i, d)) = make_float2(dqacc[r][c], dqacc[r][c + 1]);
                } else {
                    atomicAdd(qk_at(dk, i, d + 1), dkacc[r][c + 1]);
                    atomicAdd(qk_at(dq, i, d + 1), dqacc[r][c + 1]);
                    atomicAdd(qk_at(dk, i, d), dkacc[r][c]);
                    atomicAdd(qk_at(dq, i, d), dqacc[r][c]);
                }
            }
        }
    }
    __syncthreads();

    // ---- phase E: dg as the reverse cumulative sum of dG, and dbeta -----------------
    if (tid == 0) dG[C - 1] += misc[0] + gC * misc[1];
    __syncthreads();
    if (tid < C && tid < cl) {
        float acc = 0.f;
        for (int i = C - 1; i >= tid; --i) acc += dG[i];
        const size_t r = (size_t)(tok0 + tid) * H + h;
        dg[r] = g[r] < kLogGateMin ? 0.f : acc;
        dbeta[r] = dB[tid];
    }
}

template <typename IoT>
cudaError_t launch_chunked(const IoT *q, const IoT *k, const IoT *v, const float *g,
                           const float *beta, const float *h0, const int32_t *cu, int num_seqs,
                           int total_T, int Hqk, int H, const IoT *dO, const float *dSf,
                           float *dq, float *dk, float *dv, float *dg, float *dbeta, float *dh0,
                           uint8_t *ws, long long max_total, size_t base_bytes,
                           cudaStream_t stream) {
    int32_t *base = reinterpret_cast<int32_t *>(ws);
    float *recs = reinterpret_cast<float *>(ws + base_bytes);
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void *>(bwd_prep_kernel<IoT>), (int)PB_SMEM);
    if (e == cudaSuccess)
        e = ensure_dynamic_smem(reinterpret_cast<const void *>(bwd_chains_kernel), (int)CH_SMEM);
    if (e == cudaSuccess)
        e = ensure_dynamic_smem(reinterpret_cast<const void *>(bwd_local_kernel<IoT>), (int)LB_SMEM);
    if (e != cudaSuccess) return e;
    bwd_chunk_base_kernel<<<1, 1024, 0, stream>>>(cu, num_seqs, total_T, base);
    const dim3 per_chunk((unsigned)max_total, (unsigned)H);
    const dim3 per_rows((unsigned)(num_seqs * H), D / kRowBlock);
    bwd_prep_kernel<IoT><<<per_chunk, kPrepB, PB_SMEM, stream>>>(q, k, v, g, beta, dO, cu, num_seqs,
                                                                  total_T, Hqk, H, base, recs);
    bwd_chains_kernel<<<per_rows, 2 * kChainThreads, CH_SMEM, stream>>>(
        h0, dSf, dh0, cu, num_seqs, total_T, H, base, max_total, recs);
    bwd_local_kernel<IoT><<<per_chunk, kLocalThreads, LB_SMEM, stream>>>(
        q, k, v, g, dO, cu, num_seqs, total_T, Hqk, H, base, recs, dq, dk, dv, dg, dbeta);
    return cudaGetLastError();
}

// Global chunks the records must hold: exact for equal lengths, else every
// sequence may end with a partial chunk.
long long chunk_slots(int num_seqs, int total_T, bool equal) {
    if (num_seqs <= 0 || total_T <= 0) return 0;
    if (equal) return (long long)num_seqs * ((total_T / num_seqs + C - 1) / C);
    return (long long)(total_T + C - 1) / C + num_seqs;
}

size_t base_bytes_of(int num_seqs) { return ((size_t)(num_seqs + 1) * 4 + kBaseBytes - 1) & ~(kBaseBytes - 1); }

}  // namespace

size_t chunked_backward_workspace_bytes(int num_seqs, int total_T, int H, bool equal) {
    const long long slots = chunk_slots(num_seqs, total_T, equal);
    if (slots == 0) return 0;
    return base_bytes_of(num_seqs) + (size_t)slots * H * R_FLOATS * sizeof(float);
}

cudaError_t launch_backward_chunked(const void *q, const void *k, const void *v, const float *g,
                                    const float *beta, const float *h0, const int32_t *cu,
                                    int num_seqs, int total_T, int Hqk, int H, bool bf16,
                                    const void *dO, const float *dSf, float *dq, float *dk,
                                    float *dv, float *dg, float *dbeta, float *dh0,
                                    void *workspace, cudaStream_t stream) {
    const long long slots = chunk_slots(num_seqs, total_T, cu == nullptr);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    // dq and dk: with grouped heads the value heads of a group add into them
    // with atomics (zeroed first); otherwise every row of every sequence is
    // stored once by its chunk's CTA.  dv, dg, dbeta are written once.
    if (Hqk != H) {
        const size_t nq = (size_t)total_T * Hqk * D * sizeof(float);
        cudaError_t e = cudaMemsetAsync(dq, 0, nq, stream);
        if (e == cudaSuccess) e = cudaMemsetAsync(dk, 0, nq, stream);
        if (e != cudaSuccess) return e;
    }
    const size_t bb = base_bytes_of(num_seqs);
    if (bf16)
        return launch_chunked<__nv_bfloat16>(
            static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
            static_cast<const __nv_bfloat16 *>(v), g, beta, h0, cu, num_seqs, total_T, Hqk, H,
            static_cast<const __nv_bfloat16 *>(dO), dSf, dq, dk, dv, dg, dbeta, dh0, ws, slots, bb,
            stream);
    return launch_chunked<float>(static_cast<const float *>(q), static_cast<const float *>(k),
                                 static_cast<const float *>(v), g, beta, h0, cu, num_seqs, total_T,
                                 Hqk, H, static_cast<const float *>(dO), dSf, dq, dk, dv, dg, dbeta,
                                 dh0, ws, slots, bb, stream);
}

}  // namespace gdr
