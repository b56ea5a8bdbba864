"""ctypes wrapper around the plain-C fp64 token loop (gdr_oracle.c).

TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU baseline).

The inputs are the already-rounded values the CUDA path also receives
(bf16 or fp32 q/k/v, fp32 g/beta/h0); they are widened to float64 exactly and
the recurrence is evaluated in float64 with no reordering: token by token, in
the order the Gated DeltaNet / Kimi Delta Attention equations are written
(decay, erase, write, read; see gdr_oracle.c).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def library_path() -> str:
    return _LIB


def build(force: bool = False) -> str:
    """Compile gdr_oracle.c into liboracle.so with gcc (no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math",
                               "-ffp-contract=off", "-o", tmp, _SRC, "-lpthread", "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            lib.gdr_oracle_run.argtypes = [P, P, P, P, P, P, P, I64, I64, I64, I64, I64,
                                           ctypes.c_int, P, P, ctypes.c_int]
            lib.gdr_oracle_run.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: widen exactly through float32
        x = x.detach().to("cpu").float().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def run(q, k, v, g, beta, h0=None, cu_seqlens=None, *, channel_gate: bool | None = None,
        nthreads: int | None = None):
    """Evaluate the recurrence in float64.

    q, k: [T, H_qk, d_k]; v: [T, H, d_v]; g: [T, H] (scalar gate) or
    [T, H, d_k] (channel gate); beta: [T, H]; h0: [N, H, d_v, d_k] or None
    (zeros); cu_seqlens: [N + 1] or None (one sequence of length T).  H_qk
    divides H; value head h reads query/key head h // (H // H_qk).
    Returns (o [T, H, d_v], final_state [N, H, d_v, d_k]) as float64 arrays.
    """
    q, k, v, g, beta, h0 = (_f64(x) for x in (q, k, v, g, beta, h0))
    T, Hqk, dk = q.shape
    H = v.shape[1]
    dv = v.shape[2]
    if channel_gate is None:
        channel_gate = g.ndim == 3
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = len(cu) - 1
    exp_g = (T, H, dk) if channel_gate else (T, H)
    if (k.shape != (T, Hqk, dk) or v.shape[:2] != (T, H) or g.shape != exp_g
            or beta.shape != (T, H) or Hqk < 1 or H % Hqk):
        raise ValueError("oracle: inconsistent shapes")
    if h0 is not None and h0.shape != (N, H, dv, dk):
        raise ValueError("oracle: h0 shape")
    if cu[0] != 0 or cu[-1] != T:
        raise ValueError("oracle: cu_seqlens must run from 0 to T")
    o = np.empty((T, H, dv), dtype=np.float64)
    fin = np.empty((N, H, dv, dk), dtype=np.float64)
    rc = _load().gdr_oracle_run(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                                _ptr(cu), N, H, Hqk, dk, dv, int(bool(channel_gate)),
                                _ptr(o), _ptr(fin), int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"gdr_oracle_run failed ({rc})")
    return o, fin


def run_inputs(inp, heads=None, seqs=None, nthreads=None):
    """Run on an ``Inputs`` bundle, optionally on a subset of heads / sequences.

    Heads and sequences are independent, so a subset is evaluated exactly as
    in the full problem.  Returns (o, final) for the selected subset:
    o [T_sel, H_sel, d_v] covering the selected sequences' tokens in order,
    final [N_sel, H_sel, d_v, d_k].
    """
    cu = inp.cu_seqlens.numpy().astype(np.int64)
    seqs = list(range(len(cu) - 1)) if seqs is None else list(seqs)
    heads = list(range(inp.H)) if heads is None else list(heads)
    tok = np.concatenate([np.arange(cu[s], cu[s + 1]) for s in seqs]) if seqs else np.zeros(0, np.int64)
    lens = [int(cu[s + 1] - cu[s]) for s in seqs]
    sub_cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    ti = np.asarray(tok, dtype=np.int64)
    hi = np.asarray(heads, dtype=np.int64)

    grp = inp.H // int(inp.q.shape[1])
    hq = hi // grp              # query/key head of each selected value head

    def pick(x, heads=hi):
        if hasattr(x, "detach"):
            import torch
            x = x.index_select(0, torch.from_numpy(ti)).index_select(1, torch.from_numpy(heads))
            return x.float().numpy()
        return np.asarray(x)[ti][:, heads]

    h0 = None
    if inp.h0 is not None:
        h0 = inp.h0.numpy()[np.asarray(seqs, dtype=np.int64)][:, hi]
    # one q/k head per selected value head (a replicated copy where heads share)
    return run(pick(inp.q, hq), pick(inp.k, hq), pick(inp.v), pick(inp.g), pick(inp.beta), h0, sub_cu,
               channel_gate=(inp.gate_mode == "channel"), nthreads=nthreads)
