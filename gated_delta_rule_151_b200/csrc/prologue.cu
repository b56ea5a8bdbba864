// Input-side prologue of a gated delta-rule layer, in one launch:
//
//   * a depthwise causal convolution of kernel size four over the q, k and v
//     projections of every head (the short convolution of the linear-attention
//     path, page "Qwen3.8-Flash-Next and GLM-5.3-Flash share a 3:1
//     long-context pattern", section "Kimi Delta Attention extends recurrent
//     memory control"), reading before each sequence's first token the
//     convolution state a previous call handed over, and writing the state the
//     next call (a decode continuing a prefill: page "How the New Flash Models
//     Work: Inside GLM-5.3-Flash and Qwen3.8-Flash-Next", section "Serving:
//     prefill and decode are different problems") starts from;
//   * an optional SiLU, then L2 normalisation of every q and k head over its
//     d_k channels, x / sqrt(sum x^2 + 1e-6);
//   * the write strength beta = sigmoid(x_beta) and the log-gate
//     g = -c_h softplus(x_g).
//
// The pass is HBM-bound: per token and head it reads the raw q/k/v
// projections once and writes the recurrence's q/k/v once.  Roles by block:
//
//   conv blocks   persistent blocks over (tensor, 128-channel block, 64-token
//                 tile) items.  A three-stage cp.async ring brings each tile's
//                 rows (and the three before it) into shared memory two tiles
//                 ahead of the one computed, so the bytes in flight cost no
//                 registers.  Lane l of a warp owns channels 4l..4l+3; a warp
//                 takes a run of eight consecutive tokens, reads the run's
//                 eleven window rows once, and interleaves the eight norms,
//                 xor-shuffle sums over the d_k / 4 lanes of a head.  Loads and
//                 stores are contiguous 256-byte (bf16) or 512-byte (fp32) row
//                 pieces per warp.
//   gate blocks   grid-stride over the g and beta elements.
//   state blocks  one thread per (sequence, channel) writes the three inputs
//                 before the sequence's end (falling back to the incoming
//                 state for sequences shorter than three tokens).
#include "common.cuh"
#include "internal.h"

namespace gdr {
namespace {

constexpr int kProWarps = 8;                  // warps per conv block
constexpr int kProTile = 64;                  // tokens per work item
constexpr int kProRun = kProTile / kProWarps;  // consecutive tokens per warp
// a stage: the tile's rows and the three before it, 128 channels of fp32 at most
constexpr int kProStageBytes = (kProTile + 3) * 128 * 4;
constexpr int kProStages = 3;
constexpr int kProThreads = 32 * kProWarps;
constexpr float kNormEps = 1e-6f;

struct ProArgs {
    const void *xq, *xk, *xv;
    const float *wq, *wk, *wv;
    const float *xg, *gscale, *xb;
    const float *state_in;
    float *state_out;
    const int32_t *cu;
    void *q, *k, *v;
    float *g, *beta;
    int num_seqs, total_T, Hqk, H, dk, dv;
    int Cq, Cv, Call;                     // channels of q (= of k), of v, of all three
    int nbq, nbv, nball;                  // 128-channel blocks: q (= k), v, all
    int tiles;                            // token tiles
    int conv_blocks, gate_blocks, state_blocks;
    bool channel, silu, norm;
};

__device__ __forceinline__ void load4(const float *p, float (&x)[4]) {
    const float4 a = *reinterpret_cast<const float4 *>(p);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
}

__device__ __forceinline__ void load4(const __nv_bfloat16 *p, float (&x)[4]) {
    const uint2 raw = *reinterpret_cast<const uint2 *>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
}

__device__ __forceinline__ void store4(float *p, const float (&x)[4]) {
    *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
}

__device__ __forceinline__ void store4(__nv_bfloat16 *p, const float (&x)[4]) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]);
    const __nv_bfloat162 b = __floats2bfloat162_rn(x[2], x[3]);
    uint2 raw;
    raw.x = *reinterpret_cast<const uint32_t *>(&a);
    raw.y = *reinterpret_cast<const uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = raw;
}

// Sequence holding token t: [a, b) with a <= t < b, by binary search over the
// clamped cu_seqlens (equal lengths without it).  A malformed array can give
// a range without t; the caller then treats t as having no history.
__device__ __forceinline__ int seq_of(const ProArgs &A, int t, int &a, int &b) {
    if (A.cu == nullptr) {
        const int L = A.total_T / A.num_seqs;
        const int n = t / L;
        a = n * L;
        b = a + L;
        return n;
    }
    int lo = 0, hi = A.num_seqs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) / 2;
        if (min(max(A.cu[mid], 0), A.total_T) <= t) lo = mid;
        else hi = mid - 1;
    }
    sequence_range(A.cu, lo, A.num_seqs, A.total_T, a, b);
    b += a;
    return lo;
}

__device__ __forceinline__ float silu_f(float y) { return __fdividef(y, 1.0f + __expf(-y)); }

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(
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

// One work item: (tensor, 128-channel block, token tile).
struct ProItem {
    int which, cb, t0, t1, C;
};

__device__ __forceinline__ ProItem item_of(const ProArgs &A, int item) {
    ProItem it;
    const int tile = item / A.nball, cbg = item % A.nball;
    if (cbg < A.nbq) { it.which = 0; it.cb = cbg; }
    else if (cbg < 2 * A.nbq) { it.which = 1; it.cb = cbg - A.nbq; }
    else { it.which = 2; it.cb = cbg - 2 * A.nbq; }
    it.C = it.which == 2 ? A.Cv : A.Cq;
    it.t0 = tile * kProTile;
    it.t1 = min(it.t0 + kProTile, A.total_T);
    return it;
}

// Copy rows t0-3 .. t1-1 (those inside [0, total_T)) of the item's 128
// channels into a stage: row r holds token t0 - 3 + r.
template <typename IoT>
__device__ __forceinline__ void issue_tile(const ProArgs &A, const ProItem &it, uint8_t *stage) {
    const IoT *x = static_cast<const IoT *>(it.which == 0 ? A.xq : it.which == 1 ? A.xk : A.xv);
    const int width = min(128, it.C - it.cb * 128);          // channels (multiple of 16)
    constexpr int kRowBytes = 128 * (int)sizeof(IoT);
    const int pieces = width * (int)sizeof(IoT) / 16;        // 16-byte pieces per row
    const int rows = it.t1 - it.t0 + 3;
    for (int i = threadIdx.x; i < rows * pieces; i += kProThreads) {
        const int r = i / pieces, p = i % pieces;
        const int t = it.t0 - 3 + r;
        if (t < 0) continue;
        const uint8_t *src = reinterpret_cast<const uint8_t *>(x + (size_t)t * it.C + it.cb * 128);
        cp_async16(stage + r * kRowBytes + 16 * p, src + 16 * p);
    }
}

__device__ __forceinline__ void lds4(const float *p, float (&x)[4]) { load4(p, x); }
__device__ __forceinline__ void lds4(const __nv_bfloat16 *p, float (&x)[4]) { load4(p, x); }

// Outputs of the item's tokens: warp w takes the kProRun consecutive tokens
// t0 + kProRun w ..., loads their kProRun + 3 window rows from the stage once,
// computes the outputs in place (token s reads rows s..s+3 only, so oldest
// first frees row s), and interleaves the kProRun norms, xor-shuffle sums over
// the d_k / 4 lanes of a head.  Inputs before a token's sequence come from the
// incoming state (zeros without one).
template <typename IoT>
__device__ __forceinline__ void compute_tile(const ProArgs &A, const ProItem &it,
                                             const uint8_t *stage) {
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    const int c = it.cb * 128 + 4 * lane;
    const bool live = c < it.C;
    const bool normed = A.norm && it.which < 2;
    const int group = A.dk / 4;
    const int choff = it.which * A.Cq;
    const float *w = it.which == 0 ? A.wq : it.which == 1 ? A.wk : A.wv;
    IoT *y = static_cast<IoT *>(it.which == 0 ? A.q : it.which == 1 ? A.k : A.v);
    const IoT *rows = reinterpret_cast<const IoT *>(stage);
    const int tr = it.t0 + kProRun * warp;           // the run's first token
    if (tr >= it.t1) return;                         // warp-uniform

    float tap[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float t4[4] = {0.f, 0.f, 0.f, 0.f};
        if (live) load4(w + (size_t)(c + j) * 4, t4);
#pragma unroll
        for (int i = 0; i < 4; ++i) tap[j][i] = t4[i];
    }
    float xr[kProRun + 3][4];                        // tokens tr-3 .. tr+kProRun-1
#pragma unroll
    for (int r = 0; r < kProRun + 3; ++r) {
#pragma unroll
        for (int j = 0; j < 4; ++j) xr[r][j] = 0.f;
        if (live) lds4(rows + (tr - it.t0 + r) * 128 + 4 * lane, xr[r]);
    }
    // rows before a token's sequence: the incoming state, or zeros
    int a0, b0;
    const int n0 = seq_of(A, tr, a0, b0);
    const int te = min(tr + kProRun, it.t1);
    if (!(tr >= a0 + 3 && te <= b0)) {
#pragma unroll
        for (int s = 0; s < kProRun; ++s) {
            const int t = tr + s;
            if (t >= te) break;
            int a = a0, b = b0, n = n0;
            if (t >= b0 || t < a0) {
                n = seq_of(A, t, a, b);
                if (t < a || t >= b) a = t;          // malformed: no history
            }
            // token t's window rows s..s+3 hold tokens t-3..t; only the three
            // before t can lie before its sequence.  A row shared with a token
            // of another sequence is rewritten here for token t alone, so
            // the tokens are computed one at a time in this path.
            float win[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int tau = t - 3 + i;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float val = xr[s + i][j];
                    if (tau < a)
                        val = (A.state_in != nullptr && tau >= a - 3 && live)
                                  ? A.state_in[((size_t)n * A.Call + choff + c + j) * 3 + (tau - a + 3)]
                                  : 0.f;
                    win[i][j] = val;
                }
            }
            float o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float acc = tap[j][0] * win[0][j];
                acc = fmaf(tap[j][1], win[1][j], acc);
                acc = fmaf(tap[j][2], win[2][j], acc);
                acc = fmaf(tap[j][3], win[3][j], acc);
                o[j] = A.silu ? silu_f(acc) : acc;
            }
            if (normed) {
                float ss = o[0] * o[0];
#pragma unroll
                for (int j = 1; j < 4; ++j) ss = fmaf(o[j], o[j], ss);
                for (int off = group / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                const float r = rsqrtf(ss + kNormEps);
#pragma unroll
                for (int j = 0; j < 4; ++j) o[j] *= r;
            }
            if (live) store4(y + (size_t)t * it.C + c, o);
        }
        return;
    }
    // the whole run lies at least three tokens inside one sequence
#pragma unroll
    for (int s = 0; s < kProRun; ++s) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float acc = tap[j][0] * xr[s][j];
            acc = fmaf(tap[j][1], xr[s + 1][j], acc);
            acc = fmaf(tap[j][2], xr[s + 2][j], acc);
            acc = fmaf(tap[j][3], xr[s + 3][j], acc);
            xr[s][j] = A.silu ? silu_f(acc) : acc;
        }
    }
    if (normed) {
        float ss[kProRun];
#pragma unroll
        for (int s = 0; s < kProRun; ++s) {
            ss[s] = xr[s][0] * xr[s][0];
#pragma unroll
            for (int j = 1; j < 4; ++j) ss[s] = fmaf(xr[s][j], xr[s][j], ss[s]);
        }
        for (int off = group / 2; off > 0; off >>= 1) {
#pragma unroll
            for (int s = 0; s < kProRun; ++s) ss[s] += __shfl_xor_sync(0xffffffffu, ss[s], off);
        }
#pragma unroll
        for (int s = 0; s < kProRun; ++s) {
            const float r = rsqrtf(ss[s] + kNormEps);
#pragma unroll
            for (int j = 0; j < 4; ++j) xr[s][j] *= r;
        }
    }
    if (live) {
#pragma unroll
        for (int s = 0; s < kProRun; ++s)
            if (tr + s < te) store4(y + (size_t)(tr + s) * it.C + c, xr[s]);
    }
}

// Persistent conv blocks: a cp.async ring of kProStages tiles over the
// block's items, the copies of the next kProStages - 1 tiles in flight while
// this one is computed.
template <typename IoT>
__device__ void conv_blocks(const ProArgs &A, uint8_t *smem) {
    const int items = A.tiles * A.nball;
    const int first = blockIdx.x, stride = A.conv_blocks;
    const int mine = items > first ? (items - 1 - first) / stride + 1 : 0;
#pragma unroll
    for (int j = 0; j < kProStages - 1; ++j) {
        if (j < mine) issue_tile<IoT>(A, item_of(A, first + j * stride), smem + j * kProStageBytes);
        cp_async_commit();
    }
    for (int j = 0; j < mine; ++j) {
        const int jn = j + kProStages - 1;
        if (jn < mine)
            issue_tile<IoT>(A, item_of(A, first + jn * stride),
                            smem + (jn % kProStages) * kProStageBytes);
        cp_async_commit();
        cp_async_wait<kProStages - 1>();   // tile j has landed (groups complete in order)
        __syncthreads();
        compute_tile<IoT>(A, item_of(A, first + j * stride),
                          smem + (j % kProStages) * kProStageBytes);
        __syncthreads();
    }
}

__device__ __forceinline__ float softplus_f(float x) {
    return x > 20.f ? x : log1pf(expf(x));
}

template <typename IoT>
__global__ void __launch_bounds__(kProThreads, 2)
prologue_kernel(const __grid_constant__ ProArgs A) {
    const int bid = blockIdx.x;
    if (bid < A.conv_blocks) {
        extern __shared__ __align__(128) uint8_t smem[];
        conv_blocks<IoT>(A, smem);
        return;
    }
    if (bid < A.conv_blocks + A.gate_blocks) {
        const size_t stride = (size_t)A.gate_blocks * kProThreads;
        const size_t first = (size_t)(bid - A.conv_blocks) * kProThreads + threadIdx.x;
        const size_t nb = (size_t)A.total_T * A.H;
        const size_t ng = A.channel ? nb * A.dk : nb;
        for (size_t i = first; i < ng; i += stride) {
            const int h = A.channel ? (int)((i / A.dk) % A.H) : (int)(i % A.H);
            A.g[i] = -A.gscale[h] * softplus_f(A.xg[i]);
        }
        for (size_t i = first; i < nb; i += stride) A.beta[i] = 1.0f / (1.0f + expf(-A.xb[i]));
        return;
    }
    // convolution state out: the inputs at b-3, b-2, b-1 of every sequence
    const size_t i = (size_t)(bid - A.conv_blocks - A.gate_blocks) * kProThreads + threadIdx.x;
    if (i >= (size_t)A.num_seqs * A.Call) return;
    const int n = (int)(i / A.Call), ch = (int)(i % A.Call);
    int a = 0, len = 0;
    if (A.cu != nullptr) {
        sequence_range(A.cu, n, A.num_seqs, A.total_T, a, len);
    } else {
        len = A.total_T / A.num_seqs;
        a = n * len;
    }
    const int b = a + len;
    const void *xs = ch < A.Cq ? A.xq : ch < 2 * A.Cq ? A.xk : A.xv;
    const int C = ch < 2 * A.Cq ? A.Cq : A.Cv;
    const int c = ch < A.Cq ? ch : ch < 2 * A.Cq ? ch - A.Cq : ch - 2 * A.Cq;
    float s[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int tau = b - 3 + j;
        if (tau >= a)
            s[j] = to_f32(static_cast<const IoT *>(xs)[(size_t)tau * C + c]);
        else
            s[j] = A.state_in != nullptr ? A.state_in[i * 3 + (tau - a + 3)] : 0.f;
    }
#pragma unroll
    for (int j = 0; j < 3; ++j) A.state_out[i * 3 + j] = s[j];
}

}  // namespace

cudaError_t launch_prologue(const void *xq, const void *xk, const void *xv, const float *wq,
                            const float *wk, const float *wv, const float *xg,
                            const float *gscale, const float *xb, const float *state_in,
                            float *state_out, const int32_t *cu, int num_seqs, int total_T,
                            int Hqk, int H, int dk, int dv, bool channel, bool bf16, bool silu,
                            bool norm, void *q, void *k, void *v, float *g, float *beta,
                            cudaStream_t stream) {
    ProArgs A;
    A.xq = xq; A.xk = xk; A.xv = xv;
    A.wq = wq; A.wk = wk; A.wv = wv;
    A.xg = xg; A.gscale = gscale; A.xb = xb;
    A.state_in = state_in; A.state_out = state_out; A.cu = cu;
    A.q = q; A.k = k; A.v = v; A.g = g; A.beta = beta;
    A.num_seqs = num_seqs; A.total_T = total_T; A.Hqk = Hqk; A.H = H; A.dk = dk; A.dv = dv;
    A.Cq = Hqk * dk; A.Cv = H * dv; A.Call = 2 * A.Cq + A.Cv;
    A.nbq = (A.Cq + 127) / 128; A.nbv = (A.Cv + 127) / 128; A.nball = 2 * A.nbq + A.nbv;
    A.tiles = (total_T + kProTile - 1) / kProTile;
    A.channel = channel; A.silu = silu; A.norm = norm;
    const long long items = (long long)A.tiles * A.nball;
    if (items > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    // two resident CTAs per SM (three stages of 34 KiB each): one wave of
    // persistent blocks
    A.conv_blocks = (int)std::min<long long>(items, 2LL * sms);
    const long long gate_elems = (long long)total_T * H * (channel ? dk : 1);
    A.gate_blocks = total_T > 0 ? (int)std::min<long long>((gate_elems + kProThreads - 1) / kProThreads, 1184) : 0;
    A.state_blocks = state_out != nullptr
                         ? (int)(((long long)num_seqs * A.Call + kProThreads - 1) / kProThreads)
                         : 0;
    const long long blocks = (long long)A.conv_blocks + A.gate_blocks + A.state_blocks;
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    constexpr int smem = kProStages * kProStageBytes;
    if (bf16) {
        e = ensure_dynamic_smem(reinterpret_cast<const void *>(prologue_kernel<__nv_bfloat16>), smem);
        if (e != cudaSuccess) return e;
        prologue_kernel<__nv_bfloat16><<<(unsigned)blocks, kProThreads, smem, stream>>>(A);
    } else {
        e = ensure_dynamic_smem(reinterpret_cast<const void *>(prologue_kernel<float>), smem);
        if (e != cudaSuccess) return e;
        prologue_kernel<float><<<(unsigned)blocks, kProThreads, smem, stream>>>(A);
    }
    return cudaGetLastError();
}

}  // namespace gdr
