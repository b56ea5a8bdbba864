// C ABI of libgdr: argument validation, workspace sizing and kernel dispatch.
// Every check runs on the host before any launch; on error nothing is
// enqueued.  See include/gdr.h for the contract.
#include <cstdint>

#include "common.cuh"
#include "gdr.h"
#include "internal.h"

namespace {

bool valid_dim(int32_t d) { return d == 16 || d == 32 || d == 64 || d == 128; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool ok_ptr(const void *p) { return p != nullptr && aligned16(p); }

bool ok_opt_ptr(const void *p) { return p == nullptr || aligned16(p); }

// beta and scalar-mode g are read one element at a time: 4-byte alignment.
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bool ok_gate_ptr(const void *p, gdr_gate_mode_t mode) {
    return p != nullptr && (mode == GDR_GATE_CHANNEL ? aligned16(p) : aligned4(p));
}

bool ok_beta_ptr(const void *p) { return p != nullptr && aligned4(p); }

gdr_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? GDR_OK : GDR_ERR_CUDA; }

bool uses_tcgen05(int32_t d_k, int32_t d_v, gdr_gate_mode_t gate_mode, gdr_dtype_t io_dtype) {
    return gdr::tcgen05_prefill_available() && io_dtype == GDR_BF16 && d_k == 128 &&
           d_v == 128 && gdr::tcgen05_prefill_serves(gate_mode == GDR_GATE_CHANNEL);
}

}  // namespace

extern "C" {

const char *gdr_status_string(gdr_status_t status) {
    switch (status) {
        case GDR_OK: return "GDR_OK";
        case GDR_ERR_INVALID_ARG: return "GDR_ERR_INVALID_ARG: invalid argument";
        case GDR_ERR_UNSUPPORTED: return "GDR_ERR_UNSUPPORTED: unsupported request";
        case GDR_ERR_WORKSPACE: return "GDR_ERR_WORKSPACE: workspace missing or too small";
        case GDR_ERR_CUDA: return "GDR_ERR_CUDA: a CUDA call or kernel launch failed";
        case GDR_ERR_DEVICE_TIMEOUT: return "GDR_ERR_DEVICE_TIMEOUT: a device-side wait gave up";
    }
    return "GDR_ERR_UNKNOWN";
}

gdr_status_t gdr_prefill_path(int32_t d_k, int32_t d_v, gdr_gate_mode_t gate_mode,
                              gdr_dtype_t io_dtype, gdr_prefill_path_t *path) {
    if (path == nullptr || !valid_dim(d_k) || !valid_dim(d_v)) return GDR_ERR_INVALID_ARG;
    if (gate_mode != GDR_GATE_SCALAR && gate_mode != GDR_GATE_CHANNEL) return GDR_ERR_INVALID_ARG;
    if (io_dtype != GDR_F32 && io_dtype != GDR_BF16) return GDR_ERR_INVALID_ARG;
    *path = uses_tcgen05(d_k, d_v, gate_mode, io_dtype) ? GDR_PATH_TCGEN05 : GDR_PATH_SIMT;
    return GDR_OK;
}

gdr_status_t gdr_prefill_workspace_size(int32_t num_seqs, int32_t total_T, int32_t H,
                                        int32_t d_k, int32_t d_v, gdr_gate_mode_t gate_mode,
                                        gdr_dtype_t io_dtype, size_t *bytes) {
    gdr_prefill_path_t path;
    if (bytes == nullptr || num_seqs < 0 || total_T < 0 || H < 0) return GDR_ERR_INVALID_ARG;
    gdr_status_t st = gdr_prefill_path(d_k, d_v, gate_mode, io_dtype, &path);
    if (st != GDR_OK) return st;
    *bytes = 0;
    if (path == GDR_PATH_TCGEN05) {
        const size_t split = gdr::tcgen05_split_workspace_bytes(num_seqs, total_T, H);
        const size_t single = gdr::tcgen05_workspace_bytes(num_seqs, total_T, H);
        *bytes = split > single ? split : single;
    }
    return GDR_OK;
}

gdr_status_t gdr_prefill_plan(int32_t num_seqs, int32_t total_T, int32_t H, int32_t d_k,
                              int32_t d_v, gdr_gate_mode_t gate_mode, gdr_dtype_t io_dtype,
                              size_t workspace_bytes, gdr_prefill_path_t *path) {
    if (path == nullptr || num_seqs < 0 || total_T < 0 || H < 0) return GDR_ERR_INVALID_ARG;
    gdr_prefill_path_t family;
    gdr_status_t st = gdr_prefill_path(d_k, d_v, gate_mode, io_dtype, &family);
    if (st != GDR_OK) return st;
    *path = family;
    if (family == GDR_PATH_TCGEN05) {
        if (workspace_bytes < gdr::tcgen05_workspace_bytes(num_seqs, total_T, H))
            return GDR_ERR_WORKSPACE;
        const size_t split = gdr::tcgen05_split_workspace_bytes(num_seqs, total_T, H);
        if (split > 0 && workspace_bytes >= split) *path = GDR_PATH_TCGEN05_SPLIT;
    }
    return GDR_OK;
}

gdr_status_t gdr_prefill_chunked_gqa(const void *q, const void *k, const void *v,
                                     const float *g, const float *beta,
                                     const float *initial_state, const int32_t *cu_seqlens,
                                     int32_t num_seqs, int32_t total_T, int32_t H_qk, int32_t H,
                                     int32_t d_k, int32_t d_v, gdr_gate_mode_t gate_mode,
                                     gdr_dtype_t io_dtype, void *o, float *final_state,
                                     void *workspace, size_t workspace_bytes, void *stream) {
    if (num_seqs < 0 || total_T < 0 || H < 1 || H_qk < 1 || H % H_qk != 0)
        return GDR_ERR_INVALID_ARG;
    if (!valid_dim(d_k) || !valid_dim(d_v)) return GDR_ERR_INVALID_ARG;
    if (gate_mode != GDR_GATE_SCALAR && gate_mode != GDR_GATE_CHANNEL) return GDR_ERR_INVALID_ARG;
    if (io_dtype != GDR_F32 && io_dtype != GDR_BF16) return GDR_ERR_INVALID_ARG;
    if (num_seqs == 0 && total_T != 0) return GDR_ERR_INVALID_ARG;
    if (cu_seqlens == nullptr && num_seqs > 0 && total_T % num_seqs != 0) return GDR_ERR_INVALID_ARG;
    if (total_T > 0) {
        if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_gate_ptr(g, gate_mode) ||
            !ok_beta_ptr(beta) || !ok_ptr(o))
            return GDR_ERR_INVALID_ARG;
    } else if (!ok_opt_ptr(q) || !ok_opt_ptr(k) || !ok_opt_ptr(v) || !ok_opt_ptr(o)) {
        return GDR_ERR_INVALID_ARG;
    }
    if (!ok_opt_ptr(initial_state) || !ok_opt_ptr(final_state) || !ok_opt_ptr(cu_seqlens))
        return GDR_ERR_INVALID_ARG;
    // Element counts must stay addressable with 64-bit offsets and the
    // kernels' 32-bit token indices.
    if ((int64_t)total_T * H > (int64_t)INT32_MAX) return GDR_ERR_INVALID_ARG;

    // The single-kernel tcgen05 plan needs a few bytes; with the (larger) size
    // gdr_prefill_workspace_size reports, the chunk-parallel plan runs where it
    // applies.
    gdr_prefill_path_t plan;
    if (workspace_bytes > 0 && (workspace == nullptr || !aligned16(workspace)))
        return GDR_ERR_WORKSPACE;
    gdr_status_t st = gdr_prefill_plan(num_seqs, total_T, H, d_k, d_v, gate_mode, io_dtype,
                                       workspace == nullptr ? 0 : workspace_bytes, &plan);
    if (st != GDR_OK) return st;
    if (num_seqs == 0) return GDR_OK;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool channel = gate_mode == GDR_GATE_CHANNEL;
    if (plan == GDR_PATH_TCGEN05_SPLIT)
        return from_cuda(gdr::launch_prefill_split(q, k, v, g, beta, initial_state, cu_seqlens,
                                                    num_seqs, total_T, H_qk, H, channel, o,
                                                    final_state, workspace, s));
    if (plan == GDR_PATH_TCGEN05)
        return from_cuda(gdr::launch_prefill_tcgen05(q, k, v, g, beta, initial_state, cu_seqlens,
                                                      num_seqs, total_T, H_qk, H, channel, o,
                                                      final_state, workspace, s));
    return from_cuda(gdr::launch_prefill_simt(q, k, v, g, beta, initial_state, cu_seqlens,
                                              num_seqs, total_T, H_qk, H, d_k, d_v, channel,
                                              io_dtype == GDR_BF16, o, final_state, s));
}

gdr_status_t gdr_prefill_chunked(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const float *initial_state,
                                 const int32_t *cu_seqlens, int32_t num_seqs, int32_t total_T,
                                 int32_t H, int32_t d_k, int32_t d_v, gdr_gate_mode_t gate_mode,
                                 gdr_dtype_t io_dtype, void *o, float *final_state,
                                 void *workspace, size_t workspace_bytes, void *stream) {
    return gdr_prefill_chunked_gqa(q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, total_T,
                                   H, H, d_k, d_v, gate_mode, io_dtype, o, final_state, workspace,
                                   workspace_bytes, stream);
}

gdr_status_t gdr_prefill_check_workspace(const void *workspace, size_t workspace_bytes,
                                         void *stream) {
    if (workspace == nullptr || workspace_bytes == 0) return GDR_OK;
    if (workspace_bytes < sizeof(uint32_t) || !aligned16(workspace)) return GDR_ERR_INVALID_ARG;
    uint32_t word = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return GDR_ERR_CUDA;
    return word == 0 ? GDR_OK : GDR_ERR_DEVICE_TIMEOUT;
}

gdr_status_t gdr_decode_step_gqa(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, float *state, int32_t N, int32_t H_qk,
                                 int32_t H, int32_t d_k, int32_t d_v, gdr_gate_mode_t gate_mode,
                                 gdr_dtype_t io_dtype, void *o, void *stream) {
    if (N < 0 || H < 0 || H_qk < 1 || (H > 0 && H % H_qk != 0)) return GDR_ERR_INVALID_ARG;
    if (!valid_dim(d_k) || !valid_dim(d_v)) return GDR_ERR_INVALID_ARG;
    if (gate_mode != GDR_GATE_SCALAR && gate_mode != GDR_GATE_CHANNEL) return GDR_ERR_INVALID_ARG;
    if (io_dtype != GDR_F32 && io_dtype != GDR_BF16) return GDR_ERR_INVALID_ARG;
    if ((int64_t)N * H > (int64_t)INT32_MAX) return GDR_ERR_INVALID_ARG;
    if ((int64_t)N * H == 0) return GDR_OK;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_gate_ptr(g, gate_mode) ||
        !ok_beta_ptr(beta) || !ok_ptr(state) || !ok_ptr(o))
        return GDR_ERR_INVALID_ARG;
    return from_cuda(gdr::launch_decode_step(q, k, v, g, beta, state, N, H_qk, H, d_k, d_v,
                                             gate_mode == GDR_GATE_CHANNEL,
                                             io_dtype == GDR_BF16, o,
                                             static_cast<cudaStream_t>(stream)));
}

gdr_status_t gdr_decode_step(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, float *state, int32_t N, int32_t H, int32_t d_k,
                             int32_t d_v, gdr_gate_mode_t gate_mode, gdr_dtype_t io_dtype,
                             void *o, void *stream) {
    if (H < 0) return GDR_ERR_INVALID_ARG;
    return gdr_decode_step_gqa(q, k, v, g, beta, state, N, H > 0 ? H : 1, H, d_k, d_v, gate_mode,
                               io_dtype, o, stream);
}

gdr_status_t gdr_decode_multi(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, float *state, int32_t N, int32_t T,
                              int32_t H_qk, int32_t H, int32_t d_k, int32_t d_v,
                              gdr_gate_mode_t gate_mode, gdr_dtype_t io_dtype, void *o,
                              float *snapshots, void *stream) {
    if (N < 0 || T < 0 || T > 16 || H < 0 || H_qk < 1 || (H > 0 && H % H_qk != 0))
        return GDR_ERR_INVALID_ARG;
    if (!valid_dim(d_k) || !valid_dim(d_v)) return GDR_ERR_INVALID_ARG;
    if (gate_mode != GDR_GATE_SCALAR && gate_mode != GDR_GATE_CHANNEL) return GDR_ERR_INVALID_ARG;
    if (io_dtype != GDR_F32 && io_dtype != GDR_BF16) return GDR_ERR_INVALID_ARG;
    if ((int64_t)N * T * H > (int64_t)INT32_MAX) return GDR_ERR_INVALID_ARG;
    if ((int64_t)N * H * T == 0) return GDR_OK;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_gate_ptr(g, gate_mode) ||
        !ok_beta_ptr(beta) || !ok_ptr(state) || !ok_ptr(o) || !ok_opt_ptr(snapshots))
        return GDR_ERR_INVALID_ARG;
    return from_cuda(gdr::launch_decode_multi(q, k, v, g, beta, state, N, T, H_qk, H, d_k, d_v,
                                              gate_mode == GDR_GATE_CHANNEL,
                                              io_dtype == GDR_BF16, o, snapshots,
                                              static_cast<cudaStream_t>(stream)));
}

gdr_status_t gdr_prologue(const void *xq, const void *xk, const void *xv, const float *wq,
                          const float *wk, const float *wv, const float *xg, const float *gscale,
                          const float *xb, const float *conv_state_in, float *conv_state_out,
                          const int32_t *cu_seqlens, int32_t num_seqs, int32_t total_T,
                          int32_t H_qk, int32_t H, int32_t d_k, int32_t d_v,
                          gdr_gate_mode_t gate_mode, gdr_dtype_t io_dtype, uint32_t flags,
                          void *q, void *k, void *v, float *g, float *beta, void *stream) {
    if (num_seqs < 1 || total_T < 0 || H < 1 || H_qk < 1 || H % H_qk != 0)
        return GDR_ERR_INVALID_ARG;
    if (!valid_dim(d_k) || !valid_dim(d_v)) return GDR_ERR_INVALID_ARG;
    if (gate_mode != GDR_GATE_SCALAR && gate_mode != GDR_GATE_CHANNEL) return GDR_ERR_INVALID_ARG;
    if (io_dtype != GDR_F32 && io_dtype != GDR_BF16) return GDR_ERR_INVALID_ARG;
    if ((flags & ~(GDR_PROLOGUE_SILU | GDR_PROLOGUE_NORMALIZE_QK)) != 0) return GDR_ERR_INVALID_ARG;
    if (cu_seqlens == nullptr && total_T % num_seqs != 0) return GDR_ERR_INVALID_ARG;
    const int64_t Cq = (int64_t)H_qk * d_k, Cv = (int64_t)H * d_v, Call = 2 * Cq + Cv;
    if ((int64_t)total_T * Call > ((int64_t)1 << 40) || (int64_t)num_seqs * Call > INT32_MAX)
        return GDR_ERR_INVALID_ARG;
    if (conv_state_out != nullptr && !aligned4(conv_state_out)) return GDR_ERR_INVALID_ARG;
    if (conv_state_in != nullptr && !aligned4(conv_state_in)) return GDR_ERR_INVALID_ARG;
    if (!ok_ptr(wq) || !ok_ptr(wk) || !ok_ptr(wv)) return GDR_ERR_INVALID_ARG;
    if (total_T > 0) {
        if (!ok_ptr(xq) || !ok_ptr(xk) || !ok_ptr(xv) || !ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) ||
            !ok_gate_ptr(xg, gate_mode) || !ok_gate_ptr(g, gate_mode) || !ok_beta_ptr(xb) ||
            !ok_beta_ptr(beta) || gscale == nullptr || !aligned4(gscale))
            return GDR_ERR_INVALID_ARG;
    }
    // no output may overlap an input (the convolution reads neighbouring tokens)
    const size_t e = io_dtype == GDR_BF16 ? 2 : 4;
    const size_t T = (size_t)total_T, gsz = T * H * (gate_mode == GDR_GATE_CHANNEL ? d_k : 1) * 4;
    const size_t ssz = (size_t)num_seqs * Call * 3 * 4;
    struct Range {
        const void *p;
        size_t n;
    };
    const Range in[] = {{xq, T * Cq * e}, {xk, T * Cq * e}, {xv, T * Cv * e},
                        {wq, (size_t)Cq * 16}, {wk, (size_t)Cq * 16}, {wv, (size_t)Cv * 16},
                        {xg, gsz}, {gscale, (size_t)H * 4}, {xb, T * H * 4},
                        {conv_state_in, ssz},
                        {cu_seqlens, cu_seqlens ? ((size_t)num_seqs + 1) * 4 : 0}};
    const Range out[] = {{q, T * Cq * e}, {k, T * Cq * e}, {v, T * Cv * e}, {g, gsz},
                         {beta, T * H * 4}, {conv_state_out, ssz}};
    for (const Range &o : out) {
        if (o.p == nullptr || o.n == 0) continue;
        const uintptr_t o0 = reinterpret_cast<uintptr_t>(o.p), o1 = o0 + o.n;
        for (const Range &i : in) {
            if (i.p == nullptr || i.n == 0) continue;
            const uintptr_t i0 = reinterpret_cast<uintptr_t>(i.p), i1 = i0 + i.n;
            if (o0 < i1 && i0 < o1) return GDR_ERR_INVALID_ARG;
        }
        for (const Range &o2 : out) {
            if (&o2 == &o || o2.p == nullptr || o2.n == 0) continue;
            const uintptr_t a0 = reinterpret_cast<uintptr_t>(o2.p), a1 = a0 + o2.n;
            if (o0 < a1 && a0 < o1) return GDR_ERR_INVALID_ARG;
        }
    }
    if (total_T == 0 && conv_state_out == nullptr) return GDR_OK;
    return from_cuda(gdr::launch_prologue(
        xq, xk, xv, wq, wk, wv, xg, gscale, xb, conv_state_in, conv_state_out, cu_seqlens,
        num_seqs, total_T, H_qk, H, d_k, d_v, gate_mode == GDR_GATE_CHANNEL, io_dtype == GDR_BF16,
        (flags & GDR_PROLOGUE_SILU) != 0, (flags & GDR_PROLOGUE_NORMALIZE_QK) != 0, q, k, v, g,
        beta, static_cast<cudaStream_t>(stream)));
}

gdr_status_t gdr_prefill_fused(const void *xq, const void *xk, const void *xv, const float *wq,
                               const float *wk, const float *wv, const float *xg,
                               const float *gscale, const float *xb, const float *conv_state_in,
                               float *conv_state_out, const float *initial_state,
                               const int32_t *cu_seqlens, int32_t num_seqs, int32_t total_T,
                               int32_t H_qk, int32_t H, int32_t d_k, int32_t d_v,
                               gdr_gate_mode_t gate_mode, gdr_dtype_t io_dtype, uint32_t flags,
                               void *o, float *final_state, void *workspace,
                               size_t workspace_bytes, void *stream) {
    if (num_seqs < 1 || total_T < 0 || H < 1 || H_qk < 1 || H % H_qk != 0)
        return GDR_ERR_INVALID_ARG;
    if (!valid_dim(d_k) || !valid_dim(d_v)) return GDR_ERR_INVALID_ARG;
    if (gate_mode != GDR_GATE_SCALAR && gate_mode != GDR_GATE_CHANNEL) return GDR_ERR_INVALID_ARG;
    if (io_dtype != GDR_F32 && io_dtype != GDR_BF16) return GDR_ERR_INVALID_ARG;
    if ((flags & ~(GDR_PROLOGUE_SILU | GDR_PROLOGUE_NORMALIZE_QK)) != 0) return GDR_ERR_INVALID_ARG;
    if (cu_seqlens == nullptr && total_T % num_seqs != 0) return GDR_ERR_INVALID_ARG;
    if ((int64_t)total_T * H > (int64_t)INT32_MAX) return GDR_ERR_INVALID_ARG;
    const int64_t Cq = (int64_t)H_qk * d_k, Cv = (int64_t)H * d_v, Call = 2 * Cq + Cv;
    if ((int64_t)num_seqs * Call > INT32_MAX) return GDR_ERR_INVALID_ARG;
    if (conv_state_out != nullptr && !aligned4(conv_state_out)) return GDR_ERR_INVALID_ARG;
    if (conv_state_in != nullptr && !aligned4(conv_state_in)) return GDR_ERR_INVALID_ARG;
    if (!ok_ptr(wq) || !ok_ptr(wk) || !ok_ptr(wv)) return GDR_ERR_INVALID_ARG;
    if (!ok_opt_ptr(initial_state) || !ok_opt_ptr(final_state) || !ok_opt_ptr(cu_seqlens))
        return GDR_ERR_INVALID_ARG;
    if (total_T > 0) {
        if (!ok_ptr(xq) || !ok_ptr(xk) || !ok_ptr(xv) || !ok_ptr(o) ||
            !ok_gate_ptr(xg, gate_mode) || !ok_beta_ptr(xb) || gscale == nullptr ||
            !aligned4(gscale))
            return GDR_ERR_INVALID_ARG;
    }
    // outputs overlap no input (final_state may be initial_state itself, as
    // for gdr_prefill_chunked) and no other output
    const size_t T = (size_t)total_T;
    const size_t gsz = T * H * (gate_mode == GDR_GATE_CHANNEL ? d_k : 1) * 4;
    const size_t ssz = (size_t)num_seqs * Call * 3 * 4, hsz = (size_t)num_seqs * H * d_v * d_k * 4;
    struct Range {
        const void *p;
        size_t n;
    };
    const Range in[] = {{xq, T * Cq * 2}, {xk, T * Cq * 2}, {xv, T * Cv * 2},
                        {wq, (size_t)Cq * 16}, {wk, (size_t)Cq * 16}, {wv, (size_t)Cv * 16},
                        {xg, gsz}, {gscale, (size_t)H * 4}, {xb, T * H * 4},
                        {conv_state_in, ssz},
                        {initial_state == final_state ? nullptr : initial_state, hsz},
                        {cu_seqlens, ((size_t)num_seqs + 1) * 4}};
    const Range out[] = {{o, T * Cv * 2}, {final_state, hsz}, {conv_state_out, ssz}};
    for (const Range &r : out) {
        if (r.p == nullptr || r.n == 0) continue;
        const uintptr_t o0 = reinterpret_cast<uintptr_t>(r.p), o1 = o0 + r.n;
        for (const Range &i : in) {
            if (i.p == nullptr || i.n == 0) continue;
            const uintptr_t i0 = reinterpret_cast<uintptr_t>(i.p), i1 = i0 + i.n;
            if (o0 < i1 && i0 < o1) return GDR_ERR_INVALID_ARG;
        }
        for (const Range &r2 : out) {
            if (&r2 == &r || r2.p == nullptr || r2.n == 0) continue;
            const uintptr_t a0 = reinterpret_cast<uintptr_t>(r2.p), a1 = a0 + r2.n;
            if (o0 < a1 && a0 < o1) return GDR_ERR_INVALID_ARG;
        }
    }
    // the fused staging lives in the chunk-parallel tensor-core plan only
    if (!uses_tcgen05(d_k, d_v, gate_mode, io_dtype)) return GDR_ERR_UNSUPPORTED;
    if (workspace_bytes > 0 && (workspace == nullptr || !aligned16(workspace)))
        return GDR_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (total_T > 0) {
        gdr_prefill_path_t plan;
        gdr_status_t st = gdr_prefill_plan(num_seqs, total_T, H, d_k, d_v, gate_mode, io_dtype,
                                           workspace == nullptr ? 0 : workspace_bytes, &plan);
        if (st != GDR_OK) return st;
        if (plan != GDR_PATH_TCGEN05_SPLIT) return GDR_ERR_WORKSPACE;
    }
    cudaError_t e = gdr::launch_prologue_state(xq, xk, xv, conv_state_in, conv_state_out,
                                               cu_seqlens, num_seqs, total_T, H_qk, H, d_k, d_v,
                                               true, s);
    if (e != cudaSuccess) return GDR_ERR_CUDA;
    if (total_T == 0)   // no tokens: the states pass through (or start at zero)
        return gdr_prefill_chunked_gqa(nullptr, nullptr, nullptr, nullptr, nullptr, initial_state,
                                       cu_seqlens, num_seqs, 0, H_qk, H, d_k, d_v, gate_mode,
                                       io_dtype, nullptr, final_state, workspace, workspace_bytes,
                                       stream);
    gdr::PrologueIn pin;
    pin.xq = xq; pin.xk = xk; pin.xv = xv;
    pin.wq = wq; pin.wk = wk; pin.wv = wv;
    pin.xg = xg; pin.gscale = gscale; pin.xb = xb;
    pin.state_in = conv_state_in;
    pin.Cq = (int)Cq;
    pin.Call = (int)Call;
    pin.silu = (flags & GDR_PROLOGUE_SILU) != 0;
    pin.norm = (flags & GDR_PROLOGUE_NORMALIZE_QK) != 0;
    return from_cuda(gdr::launch_prefill_split(nullptr, nullptr, nullptr, nullptr, nullptr,
                                               initial_state, cu_seqlens, num_seqs, total_T, H_qk,
                                               H, gate_mode == GDR_GATE_CHANNEL, o, final_state,
                                               workspace, s, &pin));
}

gdr_status_t gdr_backward_workspace_size(int32_t num_seqs, int32_t total_T, int32_t H,
                                         int32_t d_k, int32_t d_v, size_t *bytes) {
    if (bytes == nullptr || num_seqs < 0 || total_T < 0 || H < 0 || !valid_dim(d_k) ||
        !valid_dim(d_v))
        return GDR_ERR_INVALID_ARG;
    *bytes = gdr::backward_workspace_bytes(num_seqs, total_T, H, d_k, d_v);
    // the chunked form (scalar gate, d_k = d_v = 128) needs more; with it the
    // gradient takes the chunked form where it applies
    if (d_k == 128 && d_v == 128) {
        const size_t chunked = gdr::chunked_backward_workspace_bytes(num_seqs, total_T, H, false);
        if (chunked > *bytes) *bytes = chunked;
    }
    return GDR_OK;
}

gdr_status_t gdr_backward(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, const float *initial_state, const int32_t *cu_seqlens,
                          int32_t num_seqs, int32_t total_T, int32_t H_qk, int32_t H, int32_t d_k,
                          int32_t d_v, gdr_gate_mode_t gate_mode, gdr_dtype_t io_dtype,
                          const void *d_o, const float *d_final_state, float *dq, float *dk,
                          float *dv, float *dg, float *dbeta, float *d_initial_state,
                          void *workspace, size_t workspace_bytes, void *stream) {
    if (num_seqs < 1 || total_T < 0 || H < 1 || H_qk < 1 || H % H_qk != 0)
        return GDR_ERR_INVALID_ARG;
    if (!valid_dim(d_k) || !valid_dim(d_v)) return GDR_ERR_INVALID_ARG;
    if (gate_mode != GDR_GATE_SCALAR && gate_mode != GDR_GATE_CHANNEL) return GDR_ERR_INVALID_ARG;
    if (io_dtype != GDR_F32 && io_dtype != GDR_BF16) return GDR_ERR_INVALID_ARG;
    if (cu_seqlens == nullptr && total_T % num_seqs != 0) return GDR_ERR_INVALID_ARG;
    if ((int64_t)num_seqs * H * ((d_v + 15) / 16) > INT32_MAX) return GDR_ERR_INVALID_ARG;
    if (!ok_opt_ptr(initial_state) || !ok_opt_ptr(d_final_state) || !ok_opt_ptr(d_initial_state))
        return GDR_ERR_INVALID_ARG;
    if (cu_seqlens != nullptr && !aligned4(cu_seqlens)) return GDR_ERR_INVALID_ARG;
    if (total_T > 0) {
        if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(d_o) || !ok_ptr(dq) || !ok_ptr(dk) ||
            !ok_ptr(dv) || !ok_gate_ptr(g, gate_mode) || !ok_gate_ptr(dg, gate_mode) ||
            !ok_beta_ptr(beta) || !ok_beta_ptr(dbeta))
            return GDR_ERR_INVALID_ARG;
    }
    // the chunked form where it applies and the workspace holds its records,
    // else the token loop
    const size_t chunked_need =
        (gate_mode == GDR_GATE_SCALAR && d_k == 128 && d_v == 128)
            ? gdr::chunked_backward_workspace_bytes(num_seqs, total_T, H, cu_seqlens == nullptr)
            : 0;
    const bool chunked = chunked_need > 0 && workspace != nullptr && workspace_bytes >= chunked_need &&
                         aligned16(workspace);
    const size_t need = chunked ? chunked_need : gdr::backward_workspace_bytes(num_seqs, total_T, H, d_k, d_v);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)))
        return GDR_ERR_WORKSPACE;
    // no output may overlap an input or another output
    const size_t e = io_dtype == GDR_BF16 ? 2 : 4, T = (size_t)total_T;
    const size_t nq = T * H_qk * d_k, nv = T * H * d_v, ng = T * H * (gate_mode == GDR_GATE_CHANNEL ? d_k : 1);
    const size_t ns = (size_t)num_seqs * H * d_v * d_k * 4;
    struct Range {
        const void *p;
        size_t n;
    };
    const Range in[] = {{q, nq * e}, {k, nq * e}, {v, nv * e}, {g, ng * 4}, {beta, T * H * 4},
                        {initial_state, ns}, {d_o, nv * e}, {d_final_state, ns},
                        {cu_seqlens, cu_seqlens ? ((size_t)num_seqs + 1) * 4 : 0}};
    const Range out[] = {{dq, nq * 4}, {dk, nq * 4}, {dv, nv * 4}, {dg, ng * 4},
                         {dbeta, T * H * 4}, {d_initial_state, ns}, {workspace, need}};
    for (const Range &o : out) {
        if (o.p == nullptr || o.n == 0) continue;
        const uintptr_t o0 = reinterpret_cast<uintptr_t>(o.p), o1 = o0 + o.n;
        for (const Range &i : in) {
            if (i.p == nullptr || i.n == 0) continue;
            const uintptr_t i0 = reinterpret_cast<uintptr_t>(i.p), i1 = i0 + i.n;
            if (o0 < i1 && i0 < o1) return GDR_ERR_INVALID_ARG;
        }
        for (const Range &o2 : out) {
            if (&o2 == &o || o2.p == nullptr || o2.n == 0) continue;
            const uintptr_t a0 = reinterpret_cast<uintptr_t>(o2.p), a1 = a0 + o2.n;
            if (o0 < a1 && a0 < o1) return GDR_ERR_INVALID_ARG;
        }
    }
    if (chunked)
        return from_cuda(gdr::launch_backward_chunked(
            q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, total_T, H_qk, H,
            io_dtype == GDR_BF16, d_o, d_final_state, dq, dk, dv, dg, dbeta, d_initial_state,
            workspace, static_cast<cudaStream_t>(stream)));
    return from_cuda(gdr::launch_backward(
        q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, total_T, H_qk, H, d_k, d_v,
        gate_mode == GDR_GATE_CHANNEL, io_dtype == GDR_BF16, d_o, d_final_state, dq, dk, dv, dg,
        dbeta, d_initial_state, workspace, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
