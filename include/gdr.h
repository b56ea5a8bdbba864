/*
 * gdr.h -- C ABI of libgdr, the gated delta-rule recurrence for NVIDIA B200
 * (sm_100a).
 *
 * The recurrence (page "How the New Flash Models Work: Inside GLM-5.3-Flash
 * and Qwen3.8-Flash-Next", section "Linear attention: a fixed-size memory in
 * place of the cache", Gated DeltaNet and Kimi Delta Attention equations):
 *
 *     S_t = S_{t-1} D_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t q_t
 *
 * per (sequence, head), with S_t a d_v x d_k fp32 matrix (row r = value
 * channel r, column j = key channel j) and D_t = alpha_t I (GDR_GATE_SCALAR,
 * Gated DeltaNet: one gate per head and token) or D_t = Diag(alpha_t)
 * (GDR_GATE_CHANNEL, Kimi Delta Attention: one gate per key channel).
 * With D_t = I this is the ungated rule S_t = S_{t-1} + beta_t (v_t - S_{t-1} k_t) k_t^T
 * (page "Qwen3.8-Flash vs GLM-5.3-Flash", section "The 3:1 Blueprint").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Gates are passed as their logarithm g = log(alpha) <= 0, in fp32
 *   (gates and decays stay in high precision; page "How the New Flash Models
 *   Work", section on precision).  g = -inf (alpha = 0) is allowed and resets
 *   the state; the kernels clamp g at -20 per token (alpha >= 2e-9), which
 *   changes no result by more than 2e-9 |S|.
 * - beta is fp32, any finite value.  q and k are used as given: the library
 *   neither normalises them nor scales q.
 * - Tensors are dense, row-major and contiguous, token-major:
 *     q, k     [T, H, d_k]        io dtype
 *     v, o     [T, H, d_v]        io dtype
 *     g        [T, H]             fp32 (scalar gate)
 *              [T, H, d_k]        fp32 (channel gate)
 *     beta     [T, H]             fp32
 *     state    [N, H, d_v, d_k]   fp32
 * - d_k and d_v are each one of 16, 32, 64, 128.  q, k, v, o, the states and
 *   channel-mode g must be 16-byte aligned; beta and scalar-mode g need
 *   4-byte alignment.
 * - All pointers are DEVICE pointers owned by the caller.  The library
 *   allocates nothing, keeps no global state beyond cached kernel
 *   attributes, and never synchronises the device: work is enqueued on
 *   `stream` (a cudaStream_t passed as void*; NULL = legacy default stream)
 *   and runs asynchronously.
 * - Arguments are validated on the host before anything is launched.  On any
 *   error nothing is launched and no output is written.  Launch failures
 *   return GDR_ERR_CUDA.  Device-side faults from invalid device pointers
 *   cannot be detected by the library.
 * - Outputs must not overlap inputs, except final_state == initial_state
 *   (in-place state update), which is supported.
 */
#ifndef GDR_H
#define GDR_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GDR_API __attribute__((visibility("default")))
#else
#define GDR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDR_OK = 0,
    GDR_ERR_INVALID_ARG = 1,    /* null pointer, bad size, misalignment, ... */
    GDR_ERR_UNSUPPORTED = 2,    /* valid request this build does not serve   */
    GDR_ERR_WORKSPACE = 3,      /* workspace missing or too small            */
    GDR_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed      */
    GDR_ERR_DEVICE_TIMEOUT = 5  /* a bounded device-side wait gave up        */
} gdr_status_t;

typedef enum {
    GDR_GATE_SCALAR = 0,   /* Gated DeltaNet: g [T, H]           */
    GDR_GATE_CHANNEL = 1   /* Kimi Delta Attention: g [T, H, d_k] */
} gdr_gate_mode_t;

typedef enum {
    GDR_F32 = 0,   /* q, k, v and o in fp32     */
    GDR_BF16 = 1   /* q, k, v and o in bfloat16 */
} gdr_dtype_t;

/* Which prefill kernel(s) serve a request. */
typedef enum {
    GDR_PATH_SIMT = 0,          /* fp32 CUDA-core chunked kernel (any d, any io dtype)     */
    GDR_PATH_TCGEN05 = 1,       /* tcgen05/TMEM/TMA chunked kernel (bf16, d_k = d_v = 128):
                                   one CTA per (sequence, head) runs every chunk step     */
    GDR_PATH_TCGEN05_SPLIT = 2  /* same arithmetic as two kernels: every chunk's local
                                   operands in parallel into the workspace, then one CTA
                                   per (sequence, head) runs the state chain over them    */
} gdr_prefill_path_t;

/* Human-readable name of a status code (static storage, never NULL). */
GDR_API const char *gdr_status_string(gdr_status_t status);

/*
 * Bytes of device workspace for the fastest plan gdr_prefill_chunked has for
 * this problem (written to *bytes; may be 0).  Pure host function.
 *
 * The tcgen05 kernels take two plans.  The single-kernel plan needs 16 bytes
 * (an error word).  With at most 64 (sequence, head) pairs, the
 * chunk-parallel plan (GDR_PATH_TCGEN05_SPLIT) keeps all SMs busy; it needs
 * 90,640 bytes per (chunk, sequence, head) of its chunk records, capped at
 * 1 GiB by running long problems in windows of chunks (plus 64 KiB of state
 * per (sequence, head) between windows).  The size reported here is the
 * larger one where both apply; gdr_prefill_chunked runs the chunk-parallel
 * plan when given at least that much and the single-kernel plan when given
 * at least 16 bytes.  Both give the same results up to rounding order.
 */
GDR_API gdr_status_t gdr_prefill_workspace_size(int32_t num_seqs, int32_t total_T, int32_t H,
                                        int32_t d_k, int32_t d_v,
                                        gdr_gate_mode_t gate_mode, gdr_dtype_t io_dtype,
                                        size_t *bytes);

/* The kernel family gdr_prefill_chunked uses for this shape/dtype (host only):
 * GDR_PATH_SIMT or GDR_PATH_TCGEN05. */
GDR_API gdr_status_t gdr_prefill_path(int32_t d_k, int32_t d_v, gdr_gate_mode_t gate_mode,
                              gdr_dtype_t io_dtype, gdr_prefill_path_t *path);

/*
 * The plan gdr_prefill_chunked runs for this problem given `workspace_bytes`
 * of workspace (host only): GDR_PATH_SIMT, GDR_PATH_TCGEN05 or
 * GDR_PATH_TCGEN05_SPLIT.  GDR_ERR_WORKSPACE if that workspace is below the
 * minimum; GDR_ERR_INVALID_ARG for an invalid shape or mode.
 */
GDR_API gdr_status_t gdr_prefill_plan(int32_t num_seqs, int32_t total_T, int32_t H,
                              int32_t d_k, int32_t d_v, gdr_gate_mode_t gate_mode,
                              gdr_dtype_t io_dtype, size_t workspace_bytes,
                              gdr_prefill_path_t *path);

/*
 * Chunked prefill over packed variable-length sequences.
 *
 * Runs the recurrence over every token of every sequence and head, in
 * chunks of 64 tokens that never straddle a sequence boundary; within a chunk
 * the tokens are combined in the UT/WY form (cumulative gate products, the
 * unit-lower-triangular inverse of (I + strictly-lower(beta K K^T)) weighted by
 * the gate ratios, and the chunk contractions), and the fp32 state is carried
 * on-chip from chunk to chunk.  Results equal the token loop up to rounding.
 * The token loop is the pair of update rules on page "How the New Flash
 * Models Work: Inside GLM-5.3-Flash and Qwen3.8-Flash-Next", section "Linear
 * attention: a fixed-size memory in place of the cache": the Gated DeltaNet
 * rule (scalar gate) and the Kimi Delta Attention rule (one gate per key
 * channel), each with o_t read from the updated state.  Prefill is the phase
 * that processes a whole prompt at once (same page, section "Serving:
 * prefill and decode are different problems").
 *
 * q, k, v, g, beta   inputs, layouts above, T = total_T.
 * initial_state      [num_seqs, H, d_v, d_k] fp32, or NULL for zeros.
 * cu_seqlens         DEVICE int32 [num_seqs + 1]: cu[0] = 0, non-decreasing,
 *                    cu[num_seqs] = total_T; sequence n is tokens
 *                    [cu[n], cu[n+1]).  NULL means num_seqs equal sequences of
 *                    total_T / num_seqs tokens (total_T must divide).  The
 *                    contents cannot be checked on the host: the kernels clamp
 *                    every range into [0, total_T] and treat a negative length
 *                    as empty, so a malformed array gives wrong results but no
 *                    out-of-bounds access.
 * o                  [total_T, H, d_v] output, io dtype.
 * final_state        [num_seqs, H, d_v, d_k] fp32 state after each sequence's
 *                    last token, or NULL.  May equal initial_state.  An empty
 *                    sequence yields its initial state (or zeros).
 * workspace          device scratch, 16-byte aligned: gdr_prefill_workspace_size()
 *                    bytes run the fastest plan; fewer bytes run the plan
 *                    gdr_prefill_plan reports for them (GDR_ERR_WORKSPACE
 *                    below the minimum).  NULL allowed when the minimum is 0.
 *                    Word 0 receives the device-side error bits.
 */
GDR_API gdr_status_t gdr_prefill_chunked(const void *q, const void *k, const void *v,
                                 const float *g, const float *beta,
                                 const float *initial_state, const int32_t *cu_seqlens,
                                 int32_t num_seqs, int32_t total_T, int32_t H,
                                 int32_t d_k, int32_t d_v, gdr_gate_mode_t gate_mode,
                                 gdr_dtype_t io_dtype, void *o, float *final_state,
                                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdr_prefill_chunked with grouped query/key heads: q and k are
 * [T, H_qk, d_k] while v, o, g, beta and the states carry H value heads
 * (H_qk divides H); value head h reads query/key head h / (H / H_qk).  This
 * is the head layout of the Qwen Gated DeltaNet layer, 16 query-key heads for
 * 48 value heads (page "Qwen3.8-Flash-Next and GLM-5.3-Flash ...", section
 * "Gated DeltaNet carries most of the sequence").  H_qk == H is exactly
 * gdr_prefill_chunked.  The workspace size is the one
 * gdr_prefill_workspace_size reports for H value heads.
 */
GDR_API gdr_status_t gdr_prefill_chunked_gqa(const void *q, const void *k, const void *v,
                                     const float *g, const float *beta,
                                     const float *initial_state, const int32_t *cu_seqlens,
                                     int32_t num_seqs, int32_t total_T, int32_t H_qk, int32_t H,
                                     int32_t d_k, int32_t d_v, gdr_gate_mode_t gate_mode,
                                     gdr_dtype_t io_dtype, void *o, float *final_state,
                                     void *workspace, size_t workspace_bytes, void *stream);

/*
 * After gdr_prefill_chunked's work on `stream` has finished, reports whether a
 * bounded device-side wait in it gave up (GDR_ERR_DEVICE_TIMEOUT) or not
 * (GDR_OK).  Synchronises `stream` and copies one word from `workspace`.
 */
GDR_API gdr_status_t gdr_prefill_check_workspace(const void *workspace, size_t workspace_bytes,
                                         void *stream);

/*
 * gdr_prefill_chunked for callers that cannot allocate device memory.
 *
 * Same arguments, layouts, results and errors as gdr_prefill_chunked, minus
 * the workspace.  The published method has no counterpart to this entry
 * point: it exists for callers that may not call cudaMalloc -- code whose
 * device memory is all owned by a host framework's pool, latency-critical
 * loops where an allocation would synchronise the device, plugins with no
 * allocator of their own.  Instead of a caller-provided workspace, the
 * scratch the prefill needs lives in a fixed 256-byte device array inside
 * libgdr, present on every GPU that loads the library until the process
 * exits.  The array serves the single-kernel plans (16 bytes of workspace or
 * none); a problem whose minimum exceeds 256 bytes is rejected with
 * GDR_ERR_WORKSPACE.
 *
 * The first call on each device looks up the array's device address with
 * that device current (a one-time set-up); make that first call before any
 * stream capture on the device.  All calls share the one array and clear
 * what must start at zero themselves, so calls whose GPU work overlaps (on
 * different streams or devices sharing nothing else) race on it: serialise
 * them.  Calls no cudaMalloc, cudaFree or allocating library routine.
 *
 * The device address of the array is kept per device for the life of the
 * process: after cudaDeviceReset (or any teardown of the device's primary
 * context) the library must not be used on that device again.
 */
GDR_API gdr_status_t gdr_prefill_chunked_noalloc(const void *q, const void *k, const void *v,
                                         const float *g, const float *beta,
                                         const float *initial_state, const int32_t *cu_seqlens,
                                         int32_t num_seqs, int32_t total_T, int32_t H,
                                         int32_t d_k, int32_t d_v, gdr_gate_mode_t gate_mode,
                                         gdr_dtype_t io_dtype, void *o, float *final_state,
                                         void *stream);

/*
 * The no-alloc counterpart of gdr_prefill_check_workspace.  The published
 * method has no counterpart to it.  Synchronises `stream`, then reads the
 * error word of the fixed array gdr_prefill_chunked_noalloc uses: it returns
 * GDR_ERR_DEVICE_TIMEOUT if a bounded device-side wait of a no-alloc prefill
 * (on this device, since the previous check) gave up -- that call's outputs
 * are then not valid -- and GDR_OK otherwise.  A nonzero word is cleared
 * after it is read, so each failure is reported once.  Allocates nothing.
 */
GDR_API gdr_status_t gdr_prefill_noalloc_check(void *stream);

/*
 * Test hook for gdr_prefill_noalloc_check; the published method has no
 * counterpart to it.  Enqueues on `stream` one single-thread kernel that
 * waits on a flag nothing sets, giving up after `polls` checks (1 to 2^20,
 * about 100 ns each), and records the give-up in the no-alloc array's error
 * word exactly as a prefill kernel's bounded wait does.  It cannot hang: the
 * wait always ends.  GDR_ERR_INVALID_ARG for polls outside the range.
 */
GDR_API gdr_status_t gdr_test_noalloc_wait_timeout(uint32_t polls, void *stream);

/*
 * One decode step: one new token for each of N sequences.
 *
 * q, k [N, H, d_k], v [N, H, d_v] (io dtype); g [N, H] or [N, H, d_k] fp32;
 * beta [N, H] fp32; state [N, H, d_v, d_k] fp32, read and overwritten in place
 * with S_t; o [N, H, d_v] (io dtype) receives o_t = S_t q_t.  The state makes
 * one pass through HBM (one read, one write); the serving split that hands a
 * prefill's final state to decode (page "How the New Flash Models Work",
 * section "Serving: prefill and decode are different problems") is the
 * caller passing final_state here.
 */
GDR_API gdr_status_t gdr_decode_step(const void *q, const void *k, const void *v,
                             const float *g, const float *beta, float *state,
                             int32_t N, int32_t H, int32_t d_k, int32_t d_v,
                             gdr_gate_mode_t gate_mode, gdr_dtype_t io_dtype,
                             void *o, void *stream);

/*
 * gdr_decode_step with grouped query/key heads: q, k [N, H_qk, d_k];
 * v, o [N, H, d_v]; g, beta, state per value head (H_qk divides H); value
 * head h reads query/key head h / (H / H_qk) -- the same grouping as
 * gdr_prefill_chunked_gqa.  H_qk == H is exactly gdr_decode_step.
 */
GDR_API gdr_status_t gdr_decode_step_gqa(const void *q, const void *k, const void *v,
                                 const float *g, const float *beta, float *state, int32_t N,
                                 int32_t H_qk, int32_t H, int32_t d_k, int32_t d_v,
                                 gdr_gate_mode_t gate_mode, gdr_dtype_t io_dtype, void *o,
                                 void *stream);

/*
 * T consecutive decode steps per sequence in one pass over the state -- the
 * verification step of speculative decoding, where a draft model proposes a
 * few tokens per sequence (the pages' multi-token-prediction drafting uses
 * 4-5; page "How the New Flash Models Work", multi-token prediction
 * section).  1 <= T <= 16.
 *
 * q, k [N, T, H_qk, d_k]; v [N, T, H, d_v] (io dtype); g [N, T, H] or
 * [N, T, H, d_k]; beta [N, T, H] (fp32): token t of sequence n is row
 * n*T + t.  state [N, H, d_v, d_k] fp32 is read once and overwritten with the
 * state after all T tokens; o [N, T, H, d_v] receives every token's output.
 * The results equal T calls of gdr_decode_step_gqa (same arithmetic, same
 * order).  snapshots, if not NULL, is [N, T, H, d_v, d_k] fp32 and receives
 * the state after each token (snapshot t = state after tokens 0..t), so a
 * caller that accepts only the first m drafts restores snapshot m-1.
 */
GDR_API gdr_status_t gdr_decode_multi(const void *q, const void *k, const void *v,
                              const float *g, const float *beta, float *state, int32_t N,
                              int32_t T, int32_t H_qk, int32_t H, int32_t d_k, int32_t d_v,
                              gdr_gate_mode_t gate_mode, gdr_dtype_t io_dtype, void *o,
                              float *snapshots, void *stream);

/*
 * Input-side prologue of a gated delta-rule layer: turns the raw q/k/v
 * projections and raw gate/beta activations into the recurrence's inputs.
 *
 *  - Short causal convolution, kernel size 4 (page "Qwen3.8-Flash-Next and
 *    GLM-5.3-Flash share a 3:1 long-context pattern", section "Kimi Delta
 *    Attention extends recurrent memory control"), depthwise: each channel of
 *    x_q, x_k and x_v has its own four taps,
 *        y_t[c] = w[c][0] x_{t-3}[c] + w[c][1] x_{t-2}[c] + w[c][2] x_{t-1}[c] + w[c][3] x_t[c],
 *    causal within each sequence.  Before a sequence's first token the inputs
 *    come from conv_state_in (zeros when it is NULL); conv_state_out receives
 *    each sequence's last three inputs, the state a decode call continuing
 *    the sequence starts from (page "How the New Flash Models Work", section
 *    "Serving: prefill and decode are different problems").
 *  - Optional SiLU y <- y / (1 + e^-y) (flag GDR_PROLOGUE_SILU).
 *  - Optional L2 normalisation of every q and k head over its d_k channels,
 *    y <- y / sqrt(sum y^2 + 1e-6) (flag GDR_PROLOGUE_NORMALIZE_QK).
 *  - beta = sigmoid(x_beta); log-gate g = -gscale[h] * softplus(x_g).
 *
 * Layouts (row-major, token-major like the other entry points):
 *   xq, xk, q, k   [total_T, H_qk, d_k]   io dtype
 *   xv, v          [total_T, H, d_v]      io dtype
 *   wq, wk         [H_qk * d_k, 4]        fp32 taps; tap 3 takes the current token
 *   wv             [H * d_v, 4]           fp32
 *   xg, g          [total_T, H] (GDR_GATE_SCALAR) or [total_T, H, d_k] (GDR_GATE_CHANNEL), fp32
 *   gscale         [H]                    fp32, > 0 for a decaying gate
 *   xb, beta       [total_T, H]           fp32
 *   conv_state_*   [num_seqs, 2 H_qk d_k + H d_v, 3] fp32: channels of q, then
 *                  k, then v; per channel the three inputs before (in) or at
 *                  the end of (out) the sequence, oldest first.  Either may be
 *                  NULL; they must not overlap.
 * cu_seqlens as for gdr_prefill_chunked (NULL = num_seqs equal sequences).
 * A sequence shorter than three tokens carries part of conv_state_in over to
 * conv_state_out; an empty one copies it.  For decode, pass one token per
 * sequence (cu_seqlens NULL, total_T = num_seqs).
 * Pointers: x*, q, k, v, w* and channel-mode xg/g 16-byte aligned; the rest
 * 4-byte aligned.  Outputs must not overlap the inputs (the convolution reads
 * neighbouring tokens).  Errors: GDR_ERR_INVALID_ARG for a bad size, pointer,
 * flag or overlap, before anything is launched; GDR_ERR_CUDA on launch
 * failure.
 */
#define GDR_PROLOGUE_SILU 1u
#define GDR_PROLOGUE_NORMALIZE_QK 2u

GDR_API gdr_status_t gdr_prologue(const void *xq, const void *xk, const void *xv,
                                  const float *wq, const float *wk, const float *wv,
                                  const float *xg, const float *gscale, const float *xb,
                                  const float *conv_state_in, float *conv_state_out,
                                  const int32_t *cu_seqlens, int32_t num_seqs, int32_t total_T,
                                  int32_t H_qk, int32_t H, int32_t d_k, int32_t d_v,
                                  gdr_gate_mode_t gate_mode, gdr_dtype_t io_dtype, uint32_t flags,
                                  void *q, void *k, void *v, float *g, float *beta, void *stream);

/*
 * The prologue above fused into the chunked prefill: the raw projections go
 * in, o and the final state come out, and q, k, v, g and beta never reach
 * HBM.  The prefill's stage step applies the convolution (with the incoming
 * convolution state before each sequence's first token), the optional SiLU,
 * the q/k L2 norms and the gate and beta maps to each chunk while it stages
 * the chunk's tiles, with the same arithmetic as gdr_prologue; the result is
 * the recurrence of gdr_prefill_chunked_gqa applied to gdr_prologue's outputs
 * (page "How the New Flash Models Work", section "Serving: prefill and
 * decode are different problems": the convolution state and the recurrent
 * state are what a decode continuing the sequence starts from).
 *
 * Arguments: those of gdr_prologue (raw inputs, taps, maps, convolution
 * states, flags) followed by those of gdr_prefill_chunked_gqa's state and
 * outputs: initial_state / final_state [num_seqs, H, d_v, d_k] fp32 or NULL
 * (final_state may be initial_state itself), o [total_T, H, d_v] bf16, and
 * the workspace of gdr_prefill_workspace_size.  Served for bf16 I/O with
 * d_k = d_v = 128 on the chunk-parallel tensor-core plan only:
 * GDR_ERR_UNSUPPORTED for other shapes or types (run gdr_prologue and then
 * gdr_prefill_chunked_gqa there), GDR_ERR_WORKSPACE when the workspace is
 * smaller than gdr_prefill_workspace_size reports.  No output may overlap an
 * input or another output (GDR_ERR_INVALID_ARG).  Device-side timeouts are
 * reported by gdr_prefill_check_workspace, as for gdr_prefill_chunked.
 */
GDR_API gdr_status_t gdr_prefill_fused(const void *xq, const void *xk, const void *xv,
                                       const float *wq, const float *wk, const float *wv,
                                       const float *xg, const float *gscale, const float *xb,
                                       const float *conv_state_in, float *conv_state_out,
                                       const float *initial_state, const int32_t *cu_seqlens,
                                       int32_t num_seqs, int32_t total_T, int32_t H_qk,
                                       int32_t H, int32_t d_k, int32_t d_v,
                                       gdr_gate_mode_t gate_mode, gdr_dtype_t io_dtype,
                                       uint32_t flags, void *o, float *final_state,
                                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * Gradient of the recurrence (training).  The pages train these layers but
 * print no backward pass; this is the gradient of the rule at the top of this
 * header, for the loss
 *
 *     L = sum_t <d_o_t, o_t> + sum_n <d_final_state_n, final_state_n>
 *
 * with respect to q, k, v, g, beta and the initial state.  Inputs are those
 * of gdr_prefill_chunked_gqa (same layouts, dtypes and cu_seqlens rules);
 * d_o is [total_T, H, d_v] in the io dtype; d_final_state [N, H, d_v, d_k]
 * fp32 or NULL (zeros).  Outputs, all fp32 and overwritten:
 *   dq, dk            [total_T, H_qk, d_k]  (summed over the value heads of a group)
 *   dv                [total_T, H, d_v]
 *   dg                [total_T, H] or [total_T, H, d_k]   (zero where g was clamped at -20)
 *   dbeta             [total_T, H]
 *   d_initial_state   [N, H, d_v, d_k], or NULL to skip
 * Two forms, chosen by the workspace (16-byte aligned) the caller passes:
 *   - chunked (scalar gate, d_k = d_v = 128): chunk records of 475,648
 *     bytes per (chunk, head), 256 + slots * H * 475,648 bytes with slots =
 *     N * ceil(total_T / N / 64) for equal lengths (cu_seqlens NULL), else
 *     ceil(total_T / 64) + N.  Its products run on the tensor cores over
 *     split operands (high and low bf16 or tf32 parts, fp32 accumulation);
 *     against an fp64 evaluation the gradients agree to about 1e-5 of each
 *     tensor's largest magnitude.
 *   - per token (every other shape, or a workspace too small for the
 *     records): the state checkpointed every 16 tokens, (N + ceil(total_T /
 *     16)) * H * d_v * d_k * 4 bytes; fp32 CUDA-core arithmetic.
 * gdr_backward_workspace_size reports the larger of the two where the
 * chunked form applies by shape (it does not know the gate mode), so that
 * the workspace it reports always selects the chunked form for the scalar
 * gate.  Pointers: q, k, v, d_o, the states, dq, dk, dv and channel-mode
 * g/dg 16-byte aligned; the rest 4-byte aligned.  Outputs must not overlap
 * inputs.  Errors: GDR_ERR_INVALID_ARG (size, pointer, overlap),
 * GDR_ERR_WORKSPACE (missing or too small for the token form), GDR_ERR_CUDA;
 * nothing is launched on error.  Sums over rows or over the value heads of
 * a group use floating-point atomics, so the last bits of dq, dk, dg and
 * dbeta may differ from run to run.
 */
GDR_API gdr_status_t gdr_backward_workspace_size(int32_t num_seqs, int32_t total_T, int32_t H,
                                                 int32_t d_k, int32_t d_v, size_t *bytes);

GDR_API gdr_status_t gdr_backward(const void *q, const void *k, const void *v, const float *g,
                                  const float *beta, const float *initial_state,
                                  const int32_t *cu_seqlens, int32_t num_seqs, int32_t total_T,
                                  int32_t H_qk, int32_t H, int32_t d_k, int32_t d_v,
                                  gdr_gate_mode_t gate_mode, gdr_dtype_t io_dtype,
                                  const void *d_o, const float *d_final_state, float *dq,
                                  float *dk, float *dv, float *dg, float *dbeta,
                                  float *d_initial_state, void *workspace,
                                  size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H */
