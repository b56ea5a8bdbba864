// Host-side launchers behind the C ABI (arguments already validated).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gdr {

// H counts value heads (one state each); the Hqk query/key heads each serve
// H / Hqk consecutive value heads.
cudaError_t launch_decode_step(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, float *state, int N, int Hqk, int H, int DK,
                               int DV, bool channel, bool bf16, void *o, cudaStream_t stream);

// Gradient of the recurrence: workspace for the state checkpoints, launcher.
size_t backward_workspace_bytes(int num_seqs, int total_T, int H, int DK, int DV);
cudaError_t launch_backward(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const float *h0, const int32_t *cu, int num_seqs,
                            int total_T, int Hqk, int H, int DK, int DV, bool channel, bool bf16,
                            const void *dO, const float *dSf, float *dq, float *dk, float *dv,
                            float *dg, float *dbeta, float *dh0, void *workspace,
                            cudaStream_t stream);

// Gradient in chunked form (scalar gate, d_k = d_v = 128): workspace bytes
// (equal: the sequences have equal lengths and no cu_seqlens), launcher.
size_t chunked_backward_workspace_bytes(int num_seqs, int total_T, int H, bool equal);
cudaError_t launch_backward_chunked(const void *q, const void *k, const void *v, const float *g,
                                    const float *beta, const float *h0, const int32_t *cu,
                                    int num_seqs, int total_T, int Hqk, int H, bool bf16,
                                    const void *dO, const float *dSf, float *dq, float *dk,
                                    float *dv, float *dg, float *dbeta, float *dh0,
                                    void *workspace, cudaStream_t stream);

// Input-side prologue: short causal convolution with state, q/k
// normalisation, gate and beta maps (arguments validated by the C ABI).
cudaError_t launch_prologue(const void *xq, const void *xk, const void *xv, const float *wq,
                            const float *wk, const float *wv, const float *xg,
                            const float *gscale, const float *xb, const float *state_in,
                            float *state_out, const int32_t *cu, int num_seqs, int total_T,
                            int Hqk, int H, int dk, int dv, bool channel, bool bf16, bool silu,
                            bool norm, void *q, void *k, void *v, float *g, float *beta,
                            cudaStream_t stream);

// The convolution state handed out by the prologue alone (the last three
// inputs of every channel of every sequence), for callers that fuse the rest
// of the prologue into the prefill.
cudaError_t launch_prologue_state(const void *xq, const void *xk, const void *xv,
                                  const float *state_in, float *state_out, const int32_t *cu,
                                  int num_seqs, int total_T, int Hqk, int H, int dk, int dv,
                                  bool bf16, cudaStream_t stream);

// Raw inputs of the prologue when the prefill's prep stage applies it itself
// (bf16 projections, d_k = d_v = 128).
struct PrologueIn {
    const void *xq, *xk, *xv;      // [total_T, Hqk, 128], [total_T, Hqk, 128], [total_T, H, 128]
    const float *wq, *wk, *wv;     // taps [channels, 4], tap 3 = current token
    const float *xg, *gscale, *xb; // raw gate [T, H] or [T, H, 128], coefficient [H], raw beta [T, H]
    const float *state_in;         // [num_seqs, Call, 3] or null (zeros)
    int Cq, Call;                  // channels of q (= of k); of q, k and v together
    int silu, norm;                // flags
};

// T consecutive tokens per sequence in one pass over the state (T <= 16).
cudaError_t launch_decode_multi(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, float *state, int N, int T, int Hqk, int H,
                                int DK, int DV, bool channel, bool bf16, void *o, float *snap,
                                cudaStream_t stream);

cudaError_t launch_prefill_simt(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, const float *h0, const int32_t *cu,
                                int num_seqs, int total_T, int Hqk, int H, int DK, int DV,
                                bool channel, bool bf16, void *o, float *fin,
                                cudaStream_t stream);

size_t prefill_simt_smem_bytes(int DK, int DV);

// tcgen05 prefill: bf16 I/O, d_k = d_v = 128.
bool tcgen05_prefill_available();
bool tcgen05_prefill_serves(bool channel);
size_t tcgen05_workspace_bytes(int num_seqs, int total_T, int H);
cudaError_t launch_prefill_tcgen05(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, const float *h0, const int32_t *cu,
                                   int num_seqs, int total_T, int Hqk, int H, bool channel,
                                   void *o, float *fin, void *workspace, cudaStream_t stream);

// Two-kernel chunk-parallel plan of the tcgen05 prefill: workspace bytes it
// needs (0 when the plan does not apply to this shape), and its launcher.
size_t tcgen05_split_workspace_bytes(int num_seqs, int total_T, int H);
// With `pin`, q, k, v, g and beta are ignored: the prep kernel applies the
// prologue to pin's raw inputs while it stages each chunk.
cudaError_t launch_prefill_split(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const float *h0, const int32_t *cu,
                                 int num_seqs, int total_T, int Hqk, int H, bool channel, void *o,
                                 float *fin, void *workspace, cudaStream_t stream,
                                 const PrologueIn *pin = nullptr);

}  // namespace gdr
