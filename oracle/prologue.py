"""fp64 CPU oracle for the input-side prologue of a gated delta-rule layer.

TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU baseline).  It
shares no code with the CUDA path.

What it computes, per the pages:

* A short causal convolution of kernel size four on the linear-attention path
  (page "Qwen3.8-Flash-Next and GLM-5.3-Flash share a 3:1 long-context
  pattern", section "Kimi Delta Attention extends recurrent memory control").
  The pages give only the kernel size.  Reading taken here: depthwise (one
  four-tap filter per channel), applied separately to the q, k and v
  projections of every head, causal within each sequence.
* A convolution state that a prefill hands to the decode that continues it
  (page "How the New Flash Models Work: Inside GLM-5.3-Flash and
  Qwen3.8-Flash-Next", section "Serving: prefill and decode are different
  problems").  Reading: the last three inputs of every channel of every
  sequence; before a sequence's first token the convolution reads the state
  handed in (zeros when none is).
* An optional SiLU after the convolution (the pages name no activation; off
  unless asked for).
* L2 normalisation of q and k over each head's d_k channels, as every workload
  of the pages' recurrence assumes: x / sqrt(sum(x^2) + eps), eps = 1e-6.
* The gate and write-strength maps of the workloads: beta = sigmoid(x_beta);
  log-gate g = -c_h * softplus(x_g), with c_h > 0 one coefficient per value
  head (broadcast over the d_k channels for the per-channel gate).

Every step is written out in float64 in the order above: the convolution as
the explicit four-term sum per token, no blocking or reordering.
"""
from __future__ import annotations

import numpy as np

EPS = 1e-6
TAPS = 4


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").float().numpy()
    return np.asarray(x, dtype=np.float64)


def _ranges(cu_seqlens, num_seqs, total_T):
    if cu_seqlens is None:
        L = total_T // num_seqs
        return [(n * L, (n + 1) * L) for n in range(num_seqs)]
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    return [(int(cu[n]), int(cu[n + 1])) for n in range(len(cu) - 1)]


def causal_conv(x, w, state=None, cu_seqlens=None, num_seqs=1):
    """Depthwise causal convolution of kernel size four.

    x: [T, C] inputs; w: [C, 4] taps, w[:, 3] multiplying the current token and
    w[:, 0] the token three steps back; state: [N, C, 3] inputs before each
    sequence (oldest first) or None for zeros.
    Returns (y [T, C], state_out [N, C, 3]).
    """
    x = _f64(x)
    w = _f64(w)
    T, C = x.shape
    ranges = _ranges(cu_seqlens, num_seqs, T)
    N = len(ranges)
    s_in = np.zeros((N, C, TAPS - 1)) if state is None else _f64(state)
    y = np.zeros((T, C))
    s_out = np.zeros((N, C, TAPS - 1))
    for n, (a, b) in enumerate(ranges):
        def u(tau):   # the convolution's input at absolute token tau of sequence n
            if tau >= a:
                return x[tau]
            return s_in[n, :, tau - a + TAPS - 1]
        for t in range(a, b):
            acc = np.zeros(C)
            for i in range(TAPS):
                acc = acc + w[:, i] * u(t - (TAPS - 1) + i)
            y[t] = acc
        for j in range(TAPS - 1):
            s_out[n, :, j] = u(b - (TAPS - 1) + j)
    return y, s_out


def silu(y):
    return y / (1.0 + np.exp(-y))


def l2_normalise(y, d):
    """y: [T, heads * d]; each head's d channels divided by sqrt(sum^2 + eps)."""
    T = y.shape[0]
    h = y.reshape(T, -1, d)
    return (h / np.sqrt(np.sum(h * h, axis=-1, keepdims=True) + EPS)).reshape(T, -1)


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def softplus(x):
    return np.logaddexp(0.0, x)


def prologue(xq, xk, xv, wq, wk, wv, xg, gscale, xb, *, cu_seqlens=None, num_seqs=1,
             conv_state=None, use_silu=False, normalize_qk=True):
    """The whole prologue.

    xq, xk: [T, H_qk, d_k]; xv: [T, H, d_v]; wq, wk: [H_qk * d_k, 4];
    wv: [H * d_v, 4]; xg: [T, H] or [T, H, d_k]; gscale: [H]; xb: [T, H];
    conv_state: [N, 2 H_qk d_k + H d_v, 3] (channels q | k | v) or None.
    Returns dict q, k, v (shapes of the inputs), g, beta, conv_state_out.
    """
    xq, xk, xv = _f64(xq), _f64(xk), _f64(xv)
    T, Hqk, dk = xq.shape
    H, dv = xv.shape[1], xv.shape[2]
    Cq, Cv = Hqk * dk, H * dv
    st = None if conv_state is None else _f64(conv_state)
    parts = []
    for x, w, lo, hi in ((xq, wq, 0, Cq), (xk, wk, Cq, 2 * Cq), (xv, wv, 2 * Cq, 2 * Cq + Cv)):
        y, s = causal_conv(x.reshape(T, -1), w, None if st is None else st[:, lo:hi],
                           cu_seqlens, num_seqs)
        if use_silu:
            y = silu(y)
        parts.append((y, s))
    (yq, sq), (yk, sk), (yv, sv) = parts
    if normalize_qk:
        yq, yk = l2_normalise(yq, dk), l2_normalise(yk, dk)
    xg = _f64(xg)
    c = _f64(gscale)
    if xg.ndim == 2:
        g = -c[None, :] * softplus(xg)
    else:
        g = -c[None, :, None] * softplus(xg)
    return dict(q=yq.reshape(T, Hqk, dk), k=yk.reshape(T, Hqk, dk), v=yv.reshape(T, H, dv),
                g=g, beta=sigmoid(_f64(xb)), conv_state_out=np.concatenate([sq, sk, sv], axis=1))
