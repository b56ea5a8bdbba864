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
//   conv blocks   persistent warps, each over a contiguous range of (tensor,
//                 128-channel block, run of eight tokens) items numbered block
//                 by block, so a warp walks along one channel block run after
//                 run and carries each run's last three inputs into the next.
//                 Each warp keeps its own three-stage cp.async ring of window
//                 rows in shared memory, two runs ahead of the one it
//                 computes, so the bytes in flight cost no registers and no
//                 block barrier couples the warps.  Lane l owns channels
//                 4l..4l+3; the run's outputs are computed on the packed
//                 fp32x2 units and its eight head norms reduced together.
//                 Loads and stores are contiguous 256-byte (bf16) or 512-byte
//                 (fp32) row pieces per warp.
//   gate blocks   grid-stride over the g and beta elements.
//   state blocks  one thread per (sequence, channel) writes the three inputs
//                 before the sequence's end (falling back to the incoming
//                 state for sequences shorter than three tokens).
#include "common.cuh"
#include "internal.h"

namespace gdr {
namespace {

constexpr int kProWarps = 4;                  // warps per block
constexpr int kProRun = 8;                    // consecutive tokens per work item
static_assert(kProRun == 8, "the norm butterfly spreads eight tokens over the xor-16/8/4 steps");
constexpr int kProRows = kProRun + 3;         // a run's window rows
constexpr int kProStages = 3;                 // per-warp cp.async ring
constexpr int kProThreads = 32 * kProWarps;
// shared memory of one block: every warp's ring of window rows, 128 channels
template <typename IoT>
constexpr int pro_smem_bytes() { return kProWarps * kProStages * kProRows * 128 * (int)sizeof(IoT); }

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
    int runs;                             // runs of kProRun tokens
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

// One work item: (tensor, 128-channel block, run of kProRun tokens).  Items
// are numbered channel block by channel block, so consecutive items are
// consecutive runs of one block (and a new block starts at token 0).
struct ProItem {
    int cbg, which, cb, tr, te, C;
};

__device__ __forceinline__ ProItem item_of(const ProArgs &A, int item) {
    ProItem it;
    const int run = item % A.runs;
    it.cbg = item / A.runs;
    if (it.cbg < A.nbq) { it.which = 0; it.cb = it.cbg; }
    else if (it.cbg < 2 * A.nbq) { it.which = 1; it.cb = it.cbg - A.nbq; }
    else { it.which = 2; it.cb = it.cbg - 2 * A.nbq; }
    it.C = it.which == 2 ? A.Cv : A.Cq;
    it.tr = run * kProRun;
    it.te = min(it.tr + kProRun, A.total_T);
    return it;
}

// One warp copies the rows tr-3 .. te-1 (those inside [0, total_T)) of the
// item's 128 channels into one of its stages: row r holds token tr - 3 + r.
// Without `halo` the three rows before the run are skipped: the warp carries
// them in registers from the run before.
template <typename IoT>
__device__ __forceinline__ void issue_run(const ProArgs &A, const ProItem &it, uint8_t *stage,
                                          int lane, bool halo) {
    const IoT *x = static_cast<const IoT *>(it.which == 0 ? A.xq : it.which == 1 ? A.xk : A.xv);
    const int width = min(128, it.C - it.cb * 128);          // channels (multiple of 16)
    constexpr int kRowBytes = 128 * (int)sizeof(IoT);
    constexpr int kPieces = kRowBytes / 16;                  // 16-byte pieces of a full row
    const int pieces = width * (int)sizeof(IoT) / 16;        // of this block's rows
    const uint8_t *base = reinterpret_cast<const uint8_t *>(x + it.cb * 128);
    const size_t pitch = (size_t)it.C * sizeof(IoT);
    const int r0 = halo ? 0 : 3;
    for (int i = lane + r0 * kPieces; i < kProRows * kPieces; i += 32) {
        const int r = i / kPieces, p = i % kPieces;
        const int t = it.tr - 3 + r;
        if (t < 0 || t >= it.te || p >= pieces) continue;
        cp_async16(stage + r * kRowBytes + 16 * p, base + (size_t)t * pitch + 16 * p);
    }
}

__device__ __forceinline__ void lds4(const float *p, float (&x)[4]) { load4(p, x); }
__device__ __forceinline__ void lds4(const __nv_bfloat16 *p, float (&x)[4]) { load4(p, x); }

// Outputs of a run's tokens: the warp takes the run's window rows (the three
// before it carried from the run before unless `halo`), computes the kProRun
// outputs (token s reads rows s..s+3 only), and reduces the kProRun head norms
// together, xor-shuffle sums over the d_k / 4 lanes of a head.  Inputs before
// a token's sequence come from the incoming state (zeros without one).  On
// return rows 0..2 hold the run's last three inputs, the next run's carry.
template <typename IoT>
__device__ __forceinline__ void compute_run(const ProArgs &A, const ProItem &it,
                                            const uint8_t *stage, int lane, bool halo,
                                            const float (&tap)[4][4], float (&xr)[kProRows][4],
                                            int &n0, int &a0, int &b0) {
    const int c = it.cb * 128 + 4 * lane;
    const bool live = c < it.C;
    const bool normed = A.norm && it.which < 2;
    const int group = A.dk / 4;
    const int choff = it.which * A.Cq;
    IoT *y = static_cast<IoT *>(it.which == 0 ? A.q : it.which == 1 ? A.k : A.v);
    const IoT *rows = reinterpret_cast<const IoT *>(stage);
    const int tr = it.tr, te = it.te;

    // window rows: the three before the run from the stage (halo) or carried
    // from the run before, the run's own from the stage
#pragma unroll
    for (int r = 0; r < kProRows; ++r) {
        if (r < 3 && !halo) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) xr[r][j] = 0.f;
        if (live) lds4(rows + r * 128 + 4 * lane, xr[r]);
    }
    // rows before a token's sequence: the incoming state, or zeros
    if (!(tr >= a0 && tr < b0)) n0 = seq_of(A, tr, a0, b0);   // cached across runs
    const bool fast = tr >= a0 + 3 && te <= b0;
    if (!fast) {
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
                // the same pairing as the packed path: the two paths agree bit for bit
                const float2 lo = make_float2(o[0], o[1]), hi = make_float2(o[2], o[3]);
                const float2 q2 = __ffma2_rn(hi, hi, __fmul2_rn(lo, lo));
                float ss = q2.x + q2.y;
                for (int off = group / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                const float r = rsqrt_approx(ss + kNormEps);
#pragma unroll
                for (int j = 0; j < 4; ++j) o[j] *= r;
            }
            if (live) store4(y + (size_t)t * it.C + c, o);
        }
    } else {
    // the whole run lies at least three tokens inside one sequence: pairs of
    // channels on the packed fp32x2 units
    float2 tp[2][4];                                 // [channel pair][tap]
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i) tp[h][i] = make_float2(tap[2 * h][i], tap[2 * h + 1][i]);
    float2 xp[kProRun + 3][2];
#pragma unroll
    for (int r = 0; r < kProRun + 3; ++r) {
        xp[r][0] = make_float2(xr[r][0], xr[r][1]);
        xp[r][1] = make_float2(xr[r][2], xr[r][3]);
    }
    float ss[kProRun];
#pragma unroll
    for (int s = 0; s < kProRun; ++s) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float2 acc = __fmul2_rn(tp[h][0], xp[s][h]);
            acc = __ffma2_rn(tp[h][1], xp[s + 1][h], acc);
            acc = __ffma2_rn(tp[h][2], xp[s + 2][h], acc);
            acc = __ffma2_rn(tp[h][3], xp[s + 3][h], acc);
            xp[s][h] = A.silu ? silu2(acc) : acc;    // row s is not read again
        }
        const float2 q2 = __ffma2_rn(xp[s][1], xp[s][1], __fmul2_rn(xp[s][0], xp[s][0]));
        ss[s] = q2.x + q2.y;
    }
    if (normed) {
        float tot[kProRun];
        if (group == 32) {
            norm_sums8(ss, lane, tot);
        } else {
#pragma unroll
            for (int k = 0; k < kProRun; ++k) tot[k] = ss[k];
            for (int off = group / 2; off > 0; off >>= 1) {
#pragma unroll
                for (int k = 0; k < kProRun; ++k) tot[k] += __shfl_xor_sync(0xffffffffu, tot[k], off);
            }
        }
#pragma unroll
        for (int k = 0; k < kProRun; ++k) {
            const float r = rsqrt_approx(tot[k] + kNormEps);
            xp[k][0] = __fmul2_rn(xp[k][0], make_float2(r, r));
            xp[k][1] = __fmul2_rn(xp[k][1], make_float2(r, r));
        }
    }
    if (live) {
        IoT *out = y + (size_t)tr * it.C + c;
#pragma unroll
        for (int k = 0; k < kProRun; ++k) {
            if (tr + k < te) {
                const float o4[4] = {xp[k][0].x, xp[k][0].y, xp[k][1].x, xp[k][1].y};
                store4(out, o4);
            }
            out += it.C;
        }
    }
    }
    // carry: the inputs at tr+5 .. tr+7 are the next run's rows 0..2
#pragma unroll
    for (int r = 0; r < 3; ++r)
#pragma unroll
        for (int j = 0; j < 4; ++j) xr[r][j] = xr[kProRun + r][j];
}

// Persistent warps: warp g takes the contiguous items [g per, (g+1) per), so
// it walks along one channel block run after run (a new block starts at
// token 0) and carries each run's last three inputs into the next; only its
// first item copies the three rows before the run.  Each warp has its own
// ring of kProStages stages, the copies of its next kProStages - 1 runs in
// flight while it computes this one.  cp.async groups belong to the issuing
// thread, so a warp waits for its own copies and needs no block barrier;
// __syncwarp makes the lanes' copies visible to each other and protects a
// stage until every lane is done with it.
template <typename IoT>
__device__ void conv_warps(const ProArgs &A, uint8_t *smem) {
    constexpr int kStageBytes = kProRows * 128 * (int)sizeof(IoT);
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    uint8_t *ring = smem + warp * kProStages * kStageBytes;
    const int items = A.runs * A.nball;
    const int nw = A.conv_blocks * kProWarps;
    const int per = (items + nw - 1) / nw;
    const int lo = min((blockIdx.x * kProWarps + warp) * per, items);
    const int mine = min(lo + per, items) - lo;
#pragma unroll
    for (int j = 0; j < kProStages - 1; ++j) {
        if (j < mine) issue_run<IoT>(A, item_of(A, lo + j), ring + j * kStageBytes, lane, j == 0);
        cp_async_commit();
    }
    float tap[4][4] = {};
    float xr[kProRows][4] = {};
    int tap_cbg = -1, n0 = 0, a0 = 0, b0 = -1;   // taps and sequence range held across runs
    for (int j = 0; j < mine; ++j) {
        const int jn = j + kProStages - 1;
        if (jn < mine)
            issue_run<IoT>(A, item_of(A, lo + jn), ring + (jn % kProStages) * kStageBytes, lane,
                           false);
        cp_async_commit();
        cp_async_wait<kProStages - 1>();   // run j has landed (groups complete in order)
        __syncwarp();
        const ProItem it = item_of(A, lo + j);
        if (it.cbg != tap_cbg) {
            tap_cbg = it.cbg;
            const float *w = it.which == 0 ? A.wq : it.which == 1 ? A.wk : A.wv;
            const int c = it.cb * 128 + 4 * lane;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                float t4[4] = {0.f, 0.f, 0.f, 0.f};
                if (c < it.C) load4(w + (size_t)(c + jj) * 4, t4);
#pragma unroll
                for (int i = 0; i < 4; ++i) tap[jj][i] = t4[i];
            }
        }
        compute_run<IoT>(A, it, ring + (j % kProStages) * kStageBytes, lane, j == 0, tap, xr, n0,
                         a0, b0);
        __syncwarp();
    }
}

template <typename IoT>
__global__ void __launch_bounds__(kProThreads, 4)
prologue_kernel(const __grid_constant__ ProArgs A) {
    const int bid = blockIdx.x;
    if (bid < A.conv_blocks) {
        extern __shared__ __align__(128) uint8_t smem[];
        conv_warps<IoT>(A, smem);
        return;
    }
    if (bid < A.conv_blocks + A.gate_blocks) {
        const size_t stride = (size_t)A.gate_blocks * kProThreads;
        const size_t first = (size_t)(bid - A.conv_blocks) * kProThreads + threadIdx.x;
        const size_t nb = (size_t)A.total_T * A.H;
        const size_t ng = A.channel ? nb * A.dk : nb;
        for (size_t i = first; i < ng; i += stride) {
            const int h = A.channel ? (int)((i / A.dk) % A.H) : (int)(i % A.H);
            A.g[i] = log_gate_of(A.gscale[h], A.xg[i]);
        }
        for (size_t i = first; i < nb; i += stride) A.beta[i] = beta_of(A.xb[i]);
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

// One launch of the prologue kernel with the roles A sizes.
cudaError_t run_prologue(const ProArgs &A, bool bf16, cudaStream_t stream) {
    const long long blocks = (long long)A.conv_blocks + A.gate_blocks + A.state_blocks;
    cudaError_t e;
    if (bf16) {
        constexpr int smem = pro_smem_bytes<__nv_bfloat16>();
        e = ensure_dynamic_smem(reinterpret_cast<const void *>(prologue_kernel<__nv_bfloat16>), smem);
        if (e != cudaSuccess) return e;
        prologue_kernel<__nv_bfloat16><<<(unsigned)blocks, kProThreads, smem, stream>>>(A);
    } else {
        constexpr int smem = pro_smem_bytes<float>();
        e = ensure_dynamic_smem(reinterpret_cast<const void *>(prologue_kernel<float>), smem);
        if (e != cudaSuccess) return e;
        prologue_kernel<float><<<(unsigned)blocks, kProThreads, smem, stream>>>(A);
    }
    return cudaGetLastError();
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
    A.runs = (total_T + kProRun - 1) / kProRun;
    A.channel = channel; A.silu = silu; A.norm = norm;
    const long long items = (long long)A.runs * A.nball;
    if (items > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    // one wave of persistent warps: four resident blocks of four warps per SM
    // (shared memory allows three with fp32 rows)
    const long long per_sm = bf16 ? 4 : 3;
    A.conv_blocks = (int)std::min<long long>((items + kProWarps - 1) / kProWarps, per_sm * sms);
    const long long gate_elems = (long long)total_T * H * (channel ? dk : 1);
    A.gate_blocks = total_T > 0 ? (int)std::min<long long>((gate_elems + kProThreads - 1) / kProThreads, 1184) : 0;
    A.state_blocks = state_out != nullptr
                         ? (int)(((long long)num_seqs * A.Call + kProThreads - 1) / kProThreads)
                         : 0;
    const long long blocks = (long long)A.conv_blocks + A.gate_blocks + A.state_blocks;
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    return run_prologue(A, bf16, stream);
}

cudaError_t launch_prologue_state(const void *xq, const void *xk, const void *xv,
                                  const float *state_in, float *state_out, const int32_t *cu,
                                  int num_seqs, int total_T, int Hqk, int H, int dk, int dv,
                                  bool bf16, cudaStream_t stream) {
    ProArgs A = {};
    A.xq = xq; A.xk = xk; A.xv = xv;
    A.state_in = state_in; A.state_out = state_out; A.cu = cu;
    A.num_seqs = num_seqs; A.total_T = total_T; A.Hqk = Hqk; A.H = H; A.dk = dk; A.dv = dv;
    A.Cq = Hqk * dk; A.Cv = H * dv; A.Call = 2 * A.Cq + A.Cv;
    A.conv_blocks = 0;
    A.gate_blocks = 0;
    A.state_blocks = state_out != nullptr
                         ? (int)(((long long)num_seqs * A.Call + kProThreads - 1) / kProThreads)
                         : 0;
    if (A.state_blocks == 0) return cudaSuccess;
    return run_prologue(A, bf16, stream);
}

}  // namespace gdr
