// Chunked prefill of the gated delta rule on CUDA cores (fp32 throughout).
//
// Serves every shape and dtype the C ABI accepts (fp32 or bf16 I/O, d_k and
// d_v in {16, 32, 64, 128}); the tcgen05 kernel takes over the bf16,
// d_k = d_v = 128 case.
//
// The recurrence (page "How the New Flash Models Work: Inside GLM-5.3-Flash
// and Qwen3.8-Flash-Next", section "Linear attention: a fixed-size memory in
// place of the cache") is rearranged exactly over a chunk of C = 64 tokens.
// With S_0 the state entering the chunk, G_i the within-chunk cumulative
// log-gate (scalar, or one per key channel), and Γ_i = exp(G_i):
//
//   S_i = S_0 Γ_i + Σ_{j<=i} u_j (k_j ⊙ exp(G_i - G_j))^T
//   u_i = β_i (v_i - S_{i-1} D_i k_i)
//       = β_i (v_i - S_0 (Γ_i k_i) - Σ_{j<i} u_j k_j^T Diag(exp(G_i - G_j)) k_i)
//
// so with A_ij = β_i k_i^T Diag(exp(G_i - G_j)) k_j (j < i) and T = (I + A)^-1
// (unit lower triangular):
//
//   U   = T ( diag(β) V - diag(β) (K ⊙ Γ) S_0^T )                  [C x d_v]
//   O   = (Q ⊙ Γ) S_0^T + (P ⊙ causal) U,  P_ij = q_i^T Diag(exp(G_i - G_j)) k_j
//   S_C = S_0 Γ_C + U^T (K ⊙ exp(G_C - G))
//
// Every exponent taken is <= 0 (G is non-increasing inside a chunk), so no
// intermediate can overflow.  Rows past the end of a sequence get β = 0 and
// g = 0: their A rows, u and gate increments vanish, so they change nothing.
//
// Grid: one CTA per (value-row slab of VS <= 32 rows, head, sequence).  Rows
// of S evolve independently given K, β and the gates, so slabs need no
// communication.  The CTA keeps its S slab in shared memory for the whole
// sequence and walks the chunks in order.
#include "common.cuh"

namespace gdr {
namespace {

constexpr int C = 64;
constexpr int kSimtThreads = 256;

struct SimtLayout {
    int KS, VS1, CS;
    size_t k_off, q_off, x_off, s_off, r_off, u_off, a_off, t_off, p_off, b_off, gs_off,
        gl_off, egl_off, total;
    __host__ __device__ SimtLayout(int DK, int VS) {
        KS = DK + 1;
        VS1 = VS + 1;
        CS = C + 1;
        size_t o = 0;
        k_off = o; o += (size_t)C * KS;    // K, then K ⊙ Γ
        q_off = o; o += (size_t)C * KS;    // Q, then Q ⊙ Γ
        x_off = o; o += (size_t)C * KS;    // channel G, then K ⊙ exp(G_C - G)
        s_off = o; o += (size_t)VS * KS;   // state slab S[r][c]
        r_off = o; o += (size_t)C * VS1;   // V slab, then R
        u_off = o; o += (size_t)C * VS1;   // U
        a_off = o; o += (size_t)C * CS;    // A
        t_off = o; o += (size_t)C * CS;    // T = (I + A)^-1
        p_off = o; o += (size_t)C * CS;    // P
        b_off = o; o += C;                 // beta
        gs_off = o; o += C;                // scalar G
        gl_off = o; o += DK;               // G_C per channel
        egl_off = o; o += DK;              // exp(G_C) per channel
        total = o * sizeof(float);
    }
};

__device__ __forceinline__ void tri_index(int p, int &i, int &j) {
    int ii = (int)((sqrtf(8.f * (float)p + 1.f) - 1.f) * 0.5f);
    while (ii * (ii + 1) / 2 > p) --ii;
    while ((ii + 1) * (ii + 2) / 2 <= p) ++ii;
    i = ii;
    j = p - ii * (ii + 1) / 2;
}

template <bool CHANNEL, typename IoT>
__global__ void __launch_bounds__(kSimtThreads)
prefill_simt_kernel(const IoT *__restrict__ q, const IoT *__restrict__ k,
                    const IoT *__restrict__ v, const float *__restrict__ g,
                    const float *__restrict__ beta, const float *h0,
                    const int32_t *__restrict__ cu, int num_seqs, int total_T, int Hqk, int H,
                    int DK, int DV, int VS, int nslabs, IoT *__restrict__ o, float *fin) {
    const int slab = blockIdx.x % nslabs;
    const int h = (blockIdx.x / nslabs) % H;          // value head
    const int n = blockIdx.x / (nslabs * H);
    const int hq = h / (H / Hqk);                      // its query/key head
    const int r0 = slab * VS;
    const int nv = min(VS, DV - r0);
    const int tid = threadIdx.x;
    int t0, len;
    sequence_range(cu, n, num_seqs, total_T, t0, len);

    extern __shared__ float smem[];
    const SimtLayout L(DK, VS);
    const int KS = L.KS, VS1 = L.VS1, CS = L.CS;
    float *Ks = smem + L.k_off, *Qs = smem + L.q_off, *Xs = smem + L.x_off;
    float *Ss = smem + L.s_off, *Rs = smem + L.r_off, *Us = smem + L.u_off;
    float *As = smem + L.a_off, *Ts = smem + L.t_off, *Ps = smem + L.p_off;
    float *bs = smem + L.b_off, *gs = smem + L.gs_off, *gl = smem + L.gl_off,
          *egl = smem + L.egl_off;

    const size_t state_base = ((size_t)n * H + h) * DV * DK;
    for (int idx = tid; idx < VS * DK; idx += kSimtThreads) {
        const int r = idx / DK, c = idx % DK;
        float x = 0.f;
        if (h0 != nullptr && r < nv) x = h0[state_base + (size_t)(r0 + r) * DK + c];
        Ss[r * KS + c] = x;
    }

    for (int c0 = 0; c0 < len; c0 += C) {
        const int cl = min(C, len - c0);
        // ---- stage and mask ------------------------------------------------
        for (int idx = tid; idx < C * DK; idx += kSimtThreads) {
            const int i = idx / DK, c = idx % DK;
            const bool ok = i < cl;
            const size_t row = ((size_t)(t0 + c0 + i) * H + h);
            const size_t qrow = ((size_t)(t0 + c0 + i) * Hqk + hq);
            Ks[i * KS + c] = ok ? to_f32(k[qrow * DK + c]) : 0.f;
            Qs[i * KS + c] = ok ? to_f32(q[qrow * DK + c]) : 0.f;
            if (CHANNEL) Xs[i * KS + c] = ok ? clamp_log_gate(g[row * DK + c]) : 0.f;
        }
        for (int idx = tid; idx < C * VS; idx += kSimtThreads) {
            const int i = idx / VS, r = idx % VS;
            const size_t row = ((size_t)(t0 + c0 + i) * H + h);
            Rs[i * VS1 + r] = (i < cl && r < nv) ? to_f32(v[row * DV + r0 + r]) : 0.f;
        }
        for (int i = tid; i < C; i += kSimtThreads) {
            const size_t row = ((size_t)(t0 + c0 + i) * H + h);
            bs[i] = i < cl ? beta[row] : 0.f;
            if (!CHANNEL) gs[i] = i < cl ? clamp_log_gate(g[row]) : 0.f;
        }
        __syncthreads();
        // ---- within-chunk cumulative log-gate ---------------------------------
        if (CHANNEL) {
            for (int c = tid; c < DK; c += kSimtThreads) {
                float run = 0.f;
                for (int i = 0; i < C; ++i) {
                    run += Xs[i * KS + c];
                    Xs[i * KS + c] = run;
                }
                gl[c] = run;
                egl[c] = __expf(run);
            }
        } else if (tid == 0) {
            float run = 0.f;
            for (int i = 0; i < C; ++i) {
                run += gs[i];
                gs[i] = run;
            }
            gl[0] = run;
            egl[0] = __expf(run);
        }
        __syncthreads();
        // ---- A (strictly lower) and P (lower incl. diagonal) ------------------
        for (int p = tid; p < C * (C + 1) / 2; p += kSimtThreads) {
            int i, j;
            tri_index(p, i, j);
            float dk = 0.f, dq = 0.f;
            if (CHANNEL) {
                for (int c = 0; c < DK; ++c) {
                    const float e = __expf(Xs[i * KS + c] - Xs[j * KS + c]);
                    const float kj = Ks[j * KS + c] * e;
                    dk = fmaf(Ks[i * KS + c], kj, dk);
                    dq = fmaf(Qs[i * KS + c], kj, dq);
                }
            } else {
                for (int c = 0; c < DK; ++c) {
                    dk = fmaf(Ks[i * KS + c], Ks[j * KS + c], dk);
                    dq = fmaf(Qs[i * KS + c], Ks[j * KS + c], dq);
                }
                const float e = __expf(gs[i] - gs[j]);
                dk *= e;
                dq *= e;
            }
            As[i * CS + j] = (j < i) ? bs[i] * dk : 0.f;
            Ps[i * CS + j] = dq;
        }
        __syncthreads();
        // ---- T = (I + A)^-1 by forward substitution, one column per thread;
        //      the other threads fold the gates into K and Q meanwhile ----------
        if (tid < C) {
            const int col = tid;
            for (int i = 0; i < col; ++i) Ts[i * CS + col] = 0.f;
            Ts[col * CS + col] = 1.f;
            for (int i = col + 1; i < C; ++i) {
                float x = 0.f;
                for (int j = col; j < i; ++j) x = fmaf(As[i * CS + j], Ts[j * CS + col], x);
                Ts[i * CS + col] = -x;
            }
        } else {
            for (int idx = tid - C; idx < C * DK; idx += kSimtThreads - C) {
                const int i = idx / DK, c = idx % DK;
                const float G = CHANNEL ? Xs[i * KS + c] : gs[i];
                const float GC = CHANNEL ? gl[c] : gl[0];
                const float kk = Ks[i * KS + c];
                const float e = __expf(G);
                Ks[i * KS + c] = kk * e;                       // K ⊙ Γ
                Qs[i * KS + c] *= e;                           // Q ⊙ Γ
                Xs[i * KS + c] = kk * __expf(GC - G);          // K ⊙ exp(G_C - G)
            }
        }
        __syncthreads();
        // ---- R = diag(β) (V - (K ⊙ Γ) S_0^T) -----------------------------------
        for (int idx = tid; idx < C * VS; idx += kSimtThreads) {
            const int i = idx / VS, r = idx % VS;
            float acc = 0.f;
            for (int c = 0; c < DK; ++c) acc = fmaf(Ks[i * KS + c], Ss[r * KS + c], acc);
            Rs[i * VS1 + r] = bs[i] * (Rs[i * VS1 + r] - acc);
        }
        __syncthreads();
        // ---- U = T R -----------------------------------------------------------
        for (int idx = tid; idx < C * VS; idx += kSimtThreads) {
            const int i = idx / VS, r = idx % VS;
            float acc = 0.f;
            for (int j = 0; j <= i; ++j) acc = fmaf(Ts[i * CS + j], Rs[j * VS1 + r], acc);
            Us[i * VS1 + r] = acc;
        }
        __syncthreads();
        // ---- O = (Q ⊙ Γ) S_0^T + (P ⊙ causal) U --------------------------------
        for (int idx = tid; idx < C * VS; idx += kSimtThreads) {
            const int i = idx / VS, r = idx % VS;
            float acc = 0.f;
            for (int c = 0; c < DK; ++c) acc = fmaf(Qs[i * KS + c], Ss[r * KS + c], acc);
            for (int j = 0; j <= i; ++j) acc = fmaf(Ps[i * CS + j], Us[j * VS1 + r], acc);
            if (i < cl && r < nv)
                store_io(o + ((size_t)(t0 + c0 + i) * H + h) * DV + r0 + r, acc);
        }
        __syncthreads();
        // ---- S_C = S_0 Γ_C + U^T (K ⊙ exp(G_C - G)) ------------------------------
        for (int idx = tid; idx < VS * DK; idx += kSimtThreads) {
            const int r = idx / DK, c = idx % DK;
            float acc = Ss[r * KS + c] * (CHANNEL ? egl[c] : egl[0]);
            for (int j = 0; j < C; ++j) acc = fmaf(Us[j * VS1 + r], Xs[j * KS + c], acc);
            Ss[r * KS + c] = acc;
        }
        __syncthreads();
    }

    if (fin != nullptr) {
        for (int idx = tid; idx < nv * DK; idx += kSimtThreads) {
            const int r = idx / DK, c = idx % DK;
            fin[state_base + (size_t)(r0 + r) * DK + c] = Ss[r * KS + c];
        }
    }
}

template <bool CHANNEL, typename IoT>
cudaError_t launch_typed(const void *q, const void *k, const void *v, const float *g,
                         const float *beta, const float *h0, const int32_t *cu, int num_seqs,
                         int total_T, int Hqk, int H, int DK, int DV, void *o, float *fin,
                         cudaStream_t stream) {
    const int VS = DV < 32 ? DV : 32;
    const int nslabs = (DV + VS - 1) / VS;
    const SimtLayout L(DK, VS);
    auto kern = prefill_simt_kernel<CHANNEL, IoT>;
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void *>(kern), (int)L.total);
    if (e != cudaSuccess) return e;
    const size_t blocks = (size_t)nslabs * H * num_seqs;
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffull) return cudaErrorInvalidConfiguration;
    kern<<<(unsigned)blocks, kSimtThreads, L.total, stream>>>(
        static_cast<const IoT *>(q), static_cast<const IoT *>(k), static_cast<const IoT *>(v), g,
        beta, h0, cu, num_seqs, total_T, Hqk, H, DK, DV, VS, nslabs, static_cast<IoT *>(o), fin);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_simt(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, const float *h0, const int32_t *cu,
                                int num_seqs, int total_T, int Hqk, int H, int DK, int DV,
                                bool channel, bool bf16, void *o, float *fin,
                                cudaStream_t stream) {
    if (channel)
        return bf16 ? launch_typed<true, __nv_bfloat16>(q, k, v, g, beta, h0, cu, num_seqs, total_T, Hqk, H, DK, DV, o, fin, stream)
                    : launch_typed<true, float>(q, k, v, g, beta, h0, cu, num_seqs, total_T, Hqk, H, DK, DV, o, fin, stream);
    return bf16 ? launch_typed<false, __nv_bfloat16>(q, k, v, g, beta, h0, cu, num_seqs, total_T, Hqk, H, DK, DV, o, fin, stream)
                : launch_typed<false, float>(q, k, v, g, beta, h0, cu, num_seqs, total_T, Hqk, H, DK, DV, o, fin, stream);
}

size_t prefill_simt_smem_bytes(int DK, int DV) {
    const int VS = DV < 32 ? DV : 32;
    return SimtLayout(DK, VS).total;
}

}  // namespace gdr
