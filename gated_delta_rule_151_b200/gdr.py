"""Python binding of libgdr (ctypes).  Argument marshalling only: every step of
the recurrence runs in the library's CUDA kernels.

The functions carry the C ABI's names (include/gdr.h) and take torch CUDA
tensors; they check dtype, device and contiguity, pass raw pointers and the
current CUDA stream, and raise ``GdrError`` on any non-OK status.  There is no
fallback: if libgdr.so is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdr.so")

GDR_OK = 0
GDR_ERR_INVALID_ARG = 1
GDR_ERR_UNSUPPORTED = 2
GDR_ERR_WORKSPACE = 3
GDR_ERR_CUDA = 4
GDR_ERR_DEVICE_TIMEOUT = 5

GDR_GATE_SCALAR = 0
GDR_GATE_CHANNEL = 1
GDR_F32 = 0
GDR_BF16 = 1
GDR_PATH_SIMT = 0
GDR_PATH_TCGEN05 = 1
GDR_PATH_TCGEN05_SPLIT = 2
GDR_PROLOGUE_SILU = 1
GDR_PROLOGUE_NORMALIZE_QK = 2

# Every symbol include/gdr.h declares.
EXPORTED = ("gdr_status_string", "gdr_prefill_workspace_size", "gdr_prefill_path",
            "gdr_prefill_chunked", "gdr_prefill_check_workspace", "gdr_decode_step",
            "gdr_prefill_chunked_noalloc", "gdr_prefill_chunked_gqa", "gdr_decode_step_gqa",
            "gdr_decode_multi", "gdr_prefill_plan", "gdr_prologue", "gdr_backward",
            "gdr_backward_workspace_size", "gdr_prefill_noalloc_check",
            "gdr_test_noalloc_wait_timeout", "gdr_prefill_fused")


class GdrError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {gdr_status_string(status)}")


_lock = threading.Lock()
_lib = None


def load_library():
    """Load libgdr.so once (raises if it is missing: there is no fallback)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libgdr.so not built ({LIB_PATH}); run "
                               "`python -m gated_delta_rule_151_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        ST = ctypes.c_int
        lib.gdr_status_string.argtypes = [ST]
        lib.gdr_status_string.restype = ctypes.c_char_p
        lib.gdr_prefill_workspace_size.argtypes = [I32, I32, I32, I32, I32, ST, ST,
                                                   ctypes.POINTER(SZ)]
        lib.gdr_prefill_workspace_size.restype = ST
        lib.gdr_prefill_path.argtypes = [I32, I32, ST, ST, ctypes.POINTER(ctypes.c_int)]
        lib.gdr_prefill_path.restype = ST
        lib.gdr_prefill_plan.argtypes = [I32, I32, I32, I32, I32, ST, ST, SZ,
                                         ctypes.POINTER(ctypes.c_int)]
        lib.gdr_prefill_plan.restype = ST
        lib.gdr_prefill_chunked.argtypes = [P, P, P, P, P, P, P, I32, I32, I32, I32, I32, ST, ST,
                                            P, P, P, SZ, P]
        lib.gdr_prefill_chunked.restype = ST
        lib.gdr_prefill_check_workspace.argtypes = [P, SZ, P]
        lib.gdr_prefill_check_workspace.restype = ST
        lib.gdr_decode_step.argtypes = [P, P, P, P, P, P, I32, I32, I32, I32, ST, ST, P, P]
        lib.gdr_decode_step.restype = ST
        lib.gdr_prefill_chunked_noalloc.argtypes = [P, P, P, P, P, P, P, I32, I32, I32, I32, I32,
                                                    ST, ST, P, P, P]
        lib.gdr_prefill_chunked_noalloc.restype = ST
        lib.gdr_prefill_noalloc_check.argtypes = [P]
        lib.gdr_prefill_noalloc_check.restype = ST
        lib.gdr_test_noalloc_wait_timeout.argtypes = [ctypes.c_uint32, P]
        lib.gdr_test_noalloc_wait_timeout.restype = ST
        lib.gdr_prefill_chunked_gqa.argtypes = [P, P, P, P, P, P, P, I32, I32, I32, I32, I32, I32,
                                                ST, ST, P, P, P, SZ, P]
        lib.gdr_prefill_chunked_gqa.restype = ST
        lib.gdr_decode_step_gqa.argtypes = [P, P, P, P, P, P, I32, I32, I32, I32, I32, ST, ST, P, P]
        lib.gdr_decode_step_gqa.restype = ST
        lib.gdr_decode_multi.argtypes = [P, P, P, P, P, P, I32, I32, I32, I32, I32, I32, ST, ST, P,
                                         P, P]
        lib.gdr_decode_multi.restype = ST
        lib.gdr_prologue.argtypes = [P] * 12 + [I32] * 6 + [ST, ST, ctypes.c_uint32] + [P] * 6
        lib.gdr_prologue.restype = ST
        lib.gdr_prefill_fused.argtypes = ([P] * 13 + [I32] * 6 + [ST, ST, ctypes.c_uint32] +
                                          [P, P, P, SZ, P])
        lib.gdr_prefill_fused.restype = ST
        lib.gdr_backward_workspace_size.argtypes = [I32, I32, I32, I32, I32, ctypes.POINTER(SZ)]
        lib.gdr_backward_workspace_size.restype = ST
        lib.gdr_backward.argtypes = [P] * 7 + [I32] * 6 + [ST, ST] + [P] * 9 + [SZ, P]
        lib.gdr_backward.restype = ST
        _lib = lib
        return lib


def gdr_status_string(status: int) -> str:
    return load_library().gdr_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != GDR_OK:
        raise GdrError(status, where)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _io_code(dtype: torch.dtype) -> int:
    if dtype == torch.bfloat16:
        return GDR_BF16
    if dtype == torch.float32:
        return GDR_F32
    raise TypeError(f"io dtype must be bfloat16 or float32, got {dtype}")


def _need(t, name, dtype=None, ndim=None):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")


def gdr_prefill_workspace_size(num_seqs, total_T, H, d_k, d_v, gate_mode, io_dtype) -> int:
    out = ctypes.c_size_t(0)
    _check(load_library().gdr_prefill_workspace_size(num_seqs, total_T, H, d_k, d_v, gate_mode,
                                                     io_dtype, ctypes.byref(out)),
           "gdr_prefill_workspace_size")
    return int(out.value)


def gdr_prefill_path(d_k, d_v, gate_mode, io_dtype) -> int:
    out = ctypes.c_int(0)
    _check(load_library().gdr_prefill_path(d_k, d_v, gate_mode, io_dtype, ctypes.byref(out)),
           "gdr_prefill_path")
    return int(out.value)


def gdr_prefill_plan(num_seqs, total_T, H, d_k, d_v, gate_mode, io_dtype,
                     workspace_bytes) -> int:
    """The plan gdr_prefill_chunked runs with this much workspace:
    GDR_PATH_SIMT, GDR_PATH_TCGEN05 or GDR_PATH_TCGEN05_SPLIT."""
    out = ctypes.c_int(0)
    _check(load_library().gdr_prefill_plan(num_seqs, total_T, H, d_k, d_v, gate_mode, io_dtype,
                                           workspace_bytes, ctypes.byref(out)),
           "gdr_prefill_plan")
    return int(out.value)


def _prefill(name, q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, o, final_state,
             output_final_state, workspace, stream):
    _need(q, "q", ndim=3)
    io = q.dtype
    _need(k, "k", io, 3)
    _need(v, "v", io, 3)
    _need(beta, "beta", torch.float32, 2)
    _need(g, "g", torch.float32)
    T, Hqk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    if g.dim() == 2:
        gate = GDR_GATE_SCALAR
    elif g.dim() == 3:
        gate = GDR_GATE_CHANNEL
    else:
        raise ValueError("g must be [T, H] or [T, H, d_k]")
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
        N = cu_seqlens.numel() - 1
    else:
        N = 1 if num_seqs is None else int(num_seqs)
    if initial_state is not None:
        _need(initial_state, "initial_state", torch.float32, 4)
    if o is None:
        o = torch.empty((T, H, dv), dtype=io, device=q.device)
    _need(o, "o", io, 3)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, H, dv, dk), dtype=torch.float32, device=q.device)
    if final_state is not None:
        _need(final_state, "final_state", torch.float32, 4)
    io_code = _io_code(io)
    ws_bytes = gdr_prefill_workspace_size(N, T, H, dk, dv, gate, io_code)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    lib = load_library()
    heads = (Hqk, H) if name == "gdr_prefill_chunked_gqa" else (H,)
    if name == "gdr_prefill_chunked" and Hqk != H:
        raise ValueError("q/k and v head counts differ: use gdr_prefill_chunked_gqa")
    st = getattr(lib, name)(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state), _ptr(cu_seqlens),
        N, T, *heads, dk, dv, gate, io_code, _ptr(o), _ptr(final_state), _ptr(workspace),
        workspace.numel() if workspace is not None else 0, _stream_ptr(stream))
    _check(st, name)
    return o, final_state


def gdr_prefill_chunked(q, k, v, g, beta, initial_state=None, cu_seqlens=None, *,
                        num_seqs=None, o=None, final_state=None, output_final_state=True,
                        workspace=None, stream=None):
    """Chunked prefill (see include/gdr.h).  Returns (o, final_state).

    q, k [T, H, d_k], v [T, H, d_v] (bf16 or fp32); g [T, H] or [T, H, d_k]
    fp32; beta [T, H] fp32; initial_state [N, H, d_v, d_k] fp32 or None;
    cu_seqlens int32 [N + 1] on the device, or None with ``num_seqs`` equal
    sequences (default 1).  ``final_state`` may be given (it may be the same
    tensor as initial_state); otherwise one is allocated when
    ``output_final_state``.
    """
    return _prefill("gdr_prefill_chunked", q, k, v, g, beta, initial_state, cu_seqlens, num_seqs,
                    o, final_state, output_final_state, workspace, stream)


def gdr_prefill_chunked_gqa(q, k, v, g, beta, initial_state=None, cu_seqlens=None, *,
                            num_seqs=None, o=None, final_state=None, output_final_state=True,
                            workspace=None, stream=None):
    """Chunked prefill with grouped query/key heads: q, k [T, H_qk, d_k],
    everything else per value head [T, H, ...]; H_qk divides H."""
    return _prefill("gdr_prefill_chunked_gqa", q, k, v, g, beta, initial_state, cu_seqlens,
                    num_seqs, o, final_state, output_final_state, workspace, stream)


def gdr_prefill_check_workspace(workspace, stream=None):
    _check(load_library().gdr_prefill_check_workspace(
        _ptr(workspace), workspace.numel() if workspace is not None else 0, _stream_ptr(stream)),
        "gdr_prefill_check_workspace")


def _decode(name, q, k, v, g, beta, state, o, stream):
    _need(q, "q", ndim=3)
    io = q.dtype
    _need(k, "k", io, 3)
    _need(v, "v", io, 3)
    _need(beta, "beta", torch.float32, 2)
    _need(g, "g", torch.float32)
    _need(state, "state", torch.float32, 4)
    N, Hqk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    gate = GDR_GATE_SCALAR if g.dim() == 2 else GDR_GATE_CHANNEL
    if o is None:
        o = torch.empty((N, H, dv), dtype=io, device=q.device)
    _need(o, "o", io, 3)
    if name == "gdr_decode_step" and Hqk != H:
        raise ValueError("q/k and v head counts differ: use gdr_decode_step_gqa")
    heads = (Hqk, H) if name == "gdr_decode_step_gqa" else (H,)
    st = getattr(load_library(), name)(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                       _ptr(state), N, *heads, dk, dv, gate, _io_code(io), _ptr(o),
                                       _stream_ptr(stream))
    _check(st, name)
    return o


def gdr_decode_step(q, k, v, g, beta, state, *, o=None, stream=None):
    """One decode step (see include/gdr.h): state is updated in place.

    q, k [N, H, d_k], v [N, H, d_v] (bf16 or fp32); g [N, H] or [N, H, d_k]
    fp32; beta [N, H] fp32; state [N, H, d_v, d_k] fp32.  Returns o [N, H, d_v].
    """
    return _decode("gdr_decode_step", q, k, v, g, beta, state, o, stream)


def gdr_decode_step_gqa(q, k, v, g, beta, state, *, o=None, stream=None):
    """One decode step with grouped query/key heads: q, k [N, H_qk, d_k]."""
    return _decode("gdr_decode_step_gqa", q, k, v, g, beta, state, o, stream)


def gdr_prefill_chunked_noalloc(q, k, v, g, beta, initial_state=None, cu_seqlens=None, *,
                                num_seqs=None, o=None, final_state=None, stream=None):
    """gdr_prefill_chunked without a workspace: the library's own fixed device
    scratch is used instead (see include/gdr.h for who needs this and the
    rules that come with it).  ``o`` must be given; ``final_state`` is
    optional (None: the final state is not written, and None is returned for
    it).  gdr_prefill_noalloc_check reports a device-side wait that gave up."""
    _need(q, "q", ndim=3)
    io = q.dtype
    _need(k, "k", io, 3)
    _need(v, "v", io, 3)
    _need(beta, "beta", torch.float32, 2)
    _need(g, "g", torch.float32)
    _need(o, "o", io, 3)
    T, H, dk = q.shape
    dv = v.shape[2]
    gate = GDR_GATE_SCALAR if g.dim() == 2 else GDR_GATE_CHANNEL
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
        N = cu_seqlens.numel() - 1
    else:
        N = 1 if num_seqs is None else int(num_seqs)
    if initial_state is not None:
        _need(initial_state, "initial_state", torch.float32, 4)
    if final_state is not None:
        _need(final_state, "final_state", torch.float32, 4)
    st = load_library().gdr_prefill_chunked_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state), _ptr(cu_seqlens),
        N, T, H, dk, dv, gate, _io_code(io), _ptr(o), _ptr(final_state), _stream_ptr(stream))
    _check(st, "gdr_prefill_chunked_noalloc")
    return o, final_state


def gdr_prefill_noalloc_check(stream=None):
    """Raise GdrError(GDR_ERR_DEVICE_TIMEOUT) if a bounded device-side wait of
    a no-alloc prefill gave up since the previous check (synchronises the
    stream; the error word is cleared once read)."""
    _check(load_library().gdr_prefill_noalloc_check(_stream_ptr(stream)),
           "gdr_prefill_noalloc_check")


def gdr_decode_multi(q, k, v, g, beta, state, *, o=None, snapshots=None, stream=None):
    """T consecutive decode steps per sequence in one pass (see include/gdr.h).

    q, k [N, T, H_qk, d_k]; v [N, T, H, d_v]; g [N, T, H] or [N, T, H, d_k];
    beta [N, T, H]; state [N, H, d_v, d_k] updated in place; optional
    snapshots [N, T, H, d_v, d_k] receive the state after every token.
    Returns o [N, T, H, d_v].
    """
    _need(q, "q", ndim=4)
    io = q.dtype
    _need(k, "k", io, 4)
    _need(v, "v", io, 4)
    _need(beta, "beta", torch.float32, 3)
    _need(g, "g", torch.float32)
    _need(state, "state", torch.float32, 4)
    N, T, Hqk, dk = q.shape
    H, dv = v.shape[2], v.shape[3]
    gate = GDR_GATE_SCALAR if g.dim() == 3 else GDR_GATE_CHANNEL
    if o is None:
        o = torch.empty((N, T, H, dv), dtype=io, device=q.device)
    _need(o, "o", io, 4)
    if snapshots is not None:
        _need(snapshots, "snapshots", torch.float32, 5)
    st = load_library().gdr_decode_multi(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                         _ptr(state), N, T, Hqk, H, dk, dv, gate, _io_code(io),
                                         _ptr(o), _ptr(snapshots), _stream_ptr(stream))
    _check(st, "gdr_decode_multi")
    return o


def gdr_prologue(xq, xk, xv, wq, wk, wv, xg, gscale, xb, conv_state_in=None, cu_seqlens=None, *,
                 num_seqs=None, conv_state_out=None, silu=False, normalize_qk=True, q=None,
                 k=None, v=None, g=None, beta=None, stream=None):
    """Input-side prologue (see include/gdr.h): short causal convolution with
    state, optional SiLU, q/k L2 normalisation, beta and log-gate maps.

    xq, xk [T, H_qk, d_k]; xv [T, H, d_v] (bf16 or fp32); wq, wk [H_qk d_k, 4];
    wv [H d_v, 4]; xg [T, H] or [T, H, d_k]; gscale [H]; xb [T, H];
    conv_state_in / conv_state_out [N, 2 H_qk d_k + H d_v, 3] fp32 or None.
    Returns (q, k, v, g, beta).
    """
    _need(xq, "xq", ndim=3)
    io = xq.dtype
    _need(xk, "xk", io, 3)
    _need(xv, "xv", io, 3)
    for t, name in ((wq, "wq"), (wk, "wk"), (wv, "wv")):
        _need(t, name, torch.float32, 2)
    _need(xg, "xg", torch.float32)
    _need(gscale, "gscale", torch.float32, 1)
    _need(xb, "xb", torch.float32, 2)
    T, Hqk, dk = xq.shape
    H, dv = xv.shape[1], xv.shape[2]
    gate = GDR_GATE_SCALAR if xg.dim() == 2 else GDR_GATE_CHANNEL
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
        n = cu_seqlens.numel() - 1
    else:
        n = 1 if num_seqs is None else int(num_seqs)
    if conv_state_in is not None:
        _need(conv_state_in, "conv_state_in", torch.float32, 3)
    if conv_state_out is not None:
        _need(conv_state_out, "conv_state_out", torch.float32, 3)
    dev = xq.device
    q = torch.empty_like(xq) if q is None else q
    k = torch.empty_like(xk) if k is None else k
    v = torch.empty_like(xv) if v is None else v
    g = torch.empty(xg.shape, dtype=torch.float32, device=dev) if g is None else g
    beta = torch.empty(xb.shape, dtype=torch.float32, device=dev) if beta is None else beta
    flags = (GDR_PROLOGUE_SILU if silu else 0) | (GDR_PROLOGUE_NORMALIZE_QK if normalize_qk else 0)
    st = load_library().gdr_prologue(
        _ptr(xq), _ptr(xk), _ptr(xv), _ptr(wq), _ptr(wk), _ptr(wv), _ptr(xg), _ptr(gscale),
        _ptr(xb), _ptr(conv_state_in), _ptr(conv_state_out), _ptr(cu_seqlens), n, T, Hqk, H, dk,
        dv, gate, _io_code(io), flags, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
        _stream_ptr(stream))
    _check(st, "gdr_prologue")
    return q, k, v, g, beta


def gdr_prefill_fused(xq, xk, xv, wq, wk, wv, xg, gscale, xb, conv_state_in=None,
                      initial_state=None, cu_seqlens=None, *, num_seqs=None, conv_state_out=None,
                      silu=False, normalize_qk=True, o=None, final_state=None,
                      output_final_state=True, workspace=None, stream=None):
    """The prologue fused into the chunked prefill (see include/gdr.h):
    raw inputs as for gdr_prologue, the state and outputs as for
    gdr_prefill_chunked_gqa.  Returns (o, final_state)."""
    _need(xq, "xq", torch.bfloat16, 3)
    _need(xk, "xk", torch.bfloat16, 3)
    _need(xv, "xv", torch.bfloat16, 3)
    for t, name in ((wq, "wq"), (wk, "wk"), (wv, "wv")):
        _need(t, name, torch.float32, 2)
    _need(xg, "xg", torch.float32)
    _need(gscale, "gscale", torch.float32, 1)
    _need(xb, "xb", torch.float32, 2)
    T, Hqk, dk = xq.shape
    H, dv = xv.shape[1], xv.shape[2]
    gate = GDR_GATE_SCALAR if xg.dim() == 2 else GDR_GATE_CHANNEL
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
        N = cu_seqlens.numel() - 1
    else:
        N = 1 if num_seqs is None else int(num_seqs)
    for t, name in ((conv_state_in, "conv_state_in"), (conv_state_out, "conv_state_out")):
        if t is not None:
            _need(t, name, torch.float32, 3)
    if initial_state is not None:
        _need(initial_state, "initial_state", torch.float32, 4)
    dev = xq.device
    if o is None:
        o = torch.empty((T, H, dv), dtype=torch.bfloat16, device=dev)
    _need(o, "o", torch.bfloat16, 3)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, H, dv, dk), dtype=torch.float32, device=dev)
    if final_state is not None:
        _need(final_state, "final_state", torch.float32, 4)
    ws_bytes = gdr_prefill_workspace_size(N, T, H, dk, dv, gate, GDR_BF16)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    flags = (GDR_PROLOGUE_SILU if silu else 0) | (GDR_PROLOGUE_NORMALIZE_QK if normalize_qk else 0)
    st = load_library().gdr_prefill_fused(
        _ptr(xq), _ptr(xk), _ptr(xv), _ptr(wq), _ptr(wk), _ptr(wv), _ptr(xg), _ptr(gscale),
        _ptr(xb), _ptr(conv_state_in), _ptr(conv_state_out), _ptr(initial_state),
        _ptr(cu_seqlens), N, T, Hqk, H, dk, dv, gate, GDR_BF16, flags, _ptr(o),
        _ptr(final_state), _ptr(workspace), workspace.numel() if workspace is not None else 0,
        _stream_ptr(stream))
    _check(st, "gdr_prefill_fused")
    return o, final_state


def gdr_backward_workspace_size(num_seqs, total_T, H, d_k, d_v) -> int:
    n = ctypes.c_size_t(0)
    _check(load_library().gdr_backward_workspace_size(num_seqs, total_T, H, d_k, d_v,
                                                      ctypes.byref(n)),
           "gdr_backward_workspace_size")
    return int(n.value)


def gdr_backward(q, k, v, g, beta, initial_state=None, cu_seqlens=None, *, d_o,
                 d_final_state=None, num_seqs=None, want_d_initial_state=True, workspace=None,
                 stream=None):
    """Gradient of <d_o, o> + <d_final_state, final_state> (see include/gdr.h).

    Inputs as for gdr_prefill_chunked_gqa; d_o [T, H, d_v] in the io dtype;
    d_final_state [N, H, d_v, d_k] fp32 or None.  Returns (dq, dk, dv, dg,
    dbeta, d_initial_state) as fp32 tensors (the last None unless wanted).
    Without a workspace one of gdr_backward_workspace_size bytes is
    allocated, which selects the chunked form where it applies (scalar gate,
    d = 128); a workspace too small for its records selects the per-token
    form.
    """
    _need(q, "q", ndim=3)
    io = q.dtype
    _need(k, "k", io, 3)
    _need(v, "v", io, 3)
    _need(d_o, "d_o", io, 3)
    _need(beta, "beta", torch.float32, 2)
    _need(g, "g", torch.float32)
    T, Hqk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    gate = GDR_GATE_SCALAR if g.dim() == 2 else GDR_GATE_CHANNEL
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
        n = cu_seqlens.numel() - 1
    else:
        n = 1 if num_seqs is None else int(num_seqs)
    if initial_state is not None:
        _need(initial_state, "initial_state", torch.float32, 4)
    if d_final_state is not None:
        _need(d_final_state, "d_final_state", torch.float32, 4)
    dev = q.device
    f32 = dict(dtype=torch.float32, device=dev)
    dq = torch.empty((T, Hqk, dk), **f32)
    dk_ = torch.empty((T, Hqk, dk), **f32)
    dv_ = torch.empty((T, H, dv), **f32)
    dg = torch.empty(g.shape, **f32)
    db = torch.empty((T, H), **f32)
    dh0 = torch.empty((n, H, dv, dk), **f32) if want_d_initial_state else None
    need = gdr_backward_workspace_size(n, T, H, dk, dv)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load_library().gdr_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state), _ptr(cu_seqlens),
        n, T, Hqk, H, dk, dv, gate, _io_code(io), _ptr(d_o), _ptr(d_final_state), _ptr(dq),
        _ptr(dk_), _ptr(dv_), _ptr(dg), _ptr(db), _ptr(dh0), _ptr(workspace), wsb,
        _stream_ptr(stream))
    _check(st, "gdr_backward")
    return dq, dk_, dv_, dg, db, dh0
