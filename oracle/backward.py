"""fp64 CPU oracle for the gradient of the gated delta-rule recurrence.

TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU baseline).  It
shares no code with the CUDA path.

The pages train these layers but print no backward pass, so this is the
gradient of the forward rule itself (page "How the New Flash Models Work:
Inside GLM-5.3-Flash and Qwen3.8-Flash-Next", section "Linear attention: a
fixed-size memory in place of the cache"), written token by token.  Per
(sequence, value head), with a_t = exp(g_t) (scalar, or one per key channel)
and the state S (d_v x d_k):

    E_t = S_{t-1} Diag(a_t)          x_t = E_t k_t
    u_t = beta_t (v_t - x_t)         S_t = E_t + u_t k_t^T        o_t = S_t q_t

For the loss L = sum_t <dO_t, o_t> + <dS_final, S_T> the reverse sweep, with
dS the adjoint of S_t (dS_final after the last token), is for t = T-1 .. 0:

    dS    += dO_t q_t^T                          (o_t = S_t q_t)
    dq_t  += S_t^T dO_t
    du     = dS k_t,   dk_t += dS^T u_t          (S_t = E_t + u_t k_t^T)
    dbeta_t += (v_t - x_t) . du,   dv_t = beta_t du,   dx = -beta_t du
    dE     = dS + dx k_t^T,   dk_t += E_t^T dx   (x_t = E_t k_t)
    da     = column sums of dE * S_{t-1} (summed over all entries for a
             scalar gate),   dg_t = da * a_t     (E_t = S_{t-1} Diag(a_t))
    dS     = dE Diag(a_t)

and dh0 = dS after token 0.  Grouped heads (H_qk < H) add the value heads'
dq and dk into their shared query/key head.  Everything is float64; the
states of a sequence are kept from the forward sweep (small problems only).
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").float().numpy()
    return np.asarray(x, dtype=np.float64)


def backward(q, k, v, g, beta, h0=None, cu_seqlens=None, dO=None, dS_final=None, *,
             channel_gate=None):
    """Gradients of L = <dO, O> + <dS_final, S_final>.

    q, k: [T, H_qk, d_k]; v: [T, H, d_v]; g: [T, H] or [T, H, d_k] (log-gates);
    beta: [T, H]; h0, dS_final: [N, H, d_v, d_k] or None (zeros); dO: [T, H, d_v];
    cu_seqlens: [N + 1] or None (one sequence).
    Returns dict dq, dk, dv, dg, dbeta, dh0 (float64, shapes of the inputs;
    dh0 [N, H, d_v, d_k]).
    """
    q, k, v, g, beta, h0, dO, dSf = (_f64(x) for x in (q, k, v, g, beta, h0, dO, dS_final))
    T, Hqk, dk = q.shape
    H, dv = v.shape[1], v.shape[2]
    if channel_gate is None:
        channel_gate = g.ndim == 3
    cu = np.array([0, T]) if cu_seqlens is None else np.asarray(
        cu_seqlens.detach().cpu().numpy() if hasattr(cu_seqlens, "detach") else cu_seqlens,
        dtype=np.int64)
    N = len(cu) - 1
    grp = H // Hqk
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v),
               dg=np.zeros_like(g), dbeta=np.zeros_like(beta), dh0=np.zeros((N, H, dv, dk)))
    for n in range(N):
        a0, b0 = int(cu[n]), int(cu[n + 1])
        for h in range(H):
            hq = h // grp
            S = np.zeros((dv, dk)) if h0 is None else h0[n, h].copy()
            states = [S]
            for t in range(a0, b0):
                a = np.exp(g[t, h])                       # scalar or [d_k]
                E = S * a
                x = E @ k[t, hq]
                u = beta[t, h] * (v[t, h] - x)
                S = E + np.outer(u, k[t, hq])
                states.append(S)
            dS = np.zeros((dv, dk)) if dSf is None else dSf[n, h].copy()
            for t in range(b0 - 1, a0 - 1, -1):
                Sp, St = states[t - a0], states[t - a0 + 1]
                a = np.exp(g[t, h])
                E = Sp * a
                kt, qt = k[t, hq], q[t, hq]
                x = E @ kt
                u = beta[t, h] * (v[t, h] - x)
                do = np.zeros(dv) if dO is None else dO[t, h]
                dS = dS + np.outer(do, qt)
                out["dq"][t, hq] += St.T @ do
                du = dS @ kt
                out["dk"][t, hq] += dS.T @ u
                out["dbeta"][t, h] += (v[t, h] - x) @ du
                out["dv"][t, h] += beta[t, h] * du
                dx = -beta[t, h] * du
                dE = dS + np.outer(dx, kt)
                out["dk"][t, hq] += E.T @ dx
                if channel_gate:
                    out["dg"][t, h] += (dE * Sp).sum(axis=0) * a
                else:
                    out["dg"][t, h] += (dE * Sp).sum() * a
                dS = dE * a
            out["dh0"][n, h] = dS
    return out


def loss(o, fin, dO, dS_final):
    """The scalar the gradients belong to: <dO, O> + <dS_final, S_final>."""
    val = float(np.sum(np.asarray(o) * np.asarray(dO)))
    if dS_final is not None:
        val += float(np.sum(np.asarray(fin) * np.asarray(dS_final)))
    return val
