"""Brute-force expansion of the gated delta rule into transition matrices.

TEST INFRASTRUCTURE ONLY.  This is a second, independent formulation used to
pin the token loop; it is only practical for a handful of tokens.

The page "How the New Flash Models Work: Inside GLM-5.3-Flash and
Qwen3.8-Flash-Next" (section "Linear attention: a fixed-size memory in place
of the cache") writes one token of Gated DeltaNet / Kimi Delta Attention as

    S_t = S_{t-1} A_t + beta_t v_t k_t^T,   A_t = D_t (I - beta_t k_t k_t^T),

an affine map of S_{t-1}.  Unrolling it from S_0 gives a closed form with one
explicit d_k x d_k matrix per token and no recurrence at all:

    S_t = S_0 (A_1 A_2 ... A_t) + sum_{tau <= t} beta_tau v_tau k_tau^T (A_{tau+1} ... A_t),
    o_t = S_t q_t.

Every matrix here is built densely and multiplied out.  Arrays may hold
``fractions.Fraction`` objects (exact rational arithmetic) or float64.
The gate is passed as alpha = exp(g) itself: a scalar per token (Gated
DeltaNet, D_t = alpha_t I) or a d_k vector per token (Kimi Delta Attention,
D_t = Diag(alpha_t)).
"""
from __future__ import annotations

import numpy as np


def _eye(n, like):
    one = like.flat[0] * 0 + 1 if like.size else 1
    zero = one * 0
    m = np.empty((n, n), dtype=like.dtype)
    for i in range(n):
        for j in range(n):
            m[i, j] = one if i == j else zero
    return m


def transition(k_t, alpha_t, beta_t):
    """A_t = D_t (I - beta_t k_t k_t^T) as an explicit d_k x d_k matrix."""
    dk = k_t.shape[0]
    I = _eye(dk, k_t)
    erase = I - beta_t * np.outer(k_t, k_t)
    if np.ndim(alpha_t) == 0:
        D = I * alpha_t
    else:
        D = _eye(dk, k_t) * 0
        for j in range(dk):
            D[j, j] = alpha_t[j]
    return D.dot(erase)


def expand(q, k, v, alpha, beta, S0):
    """Closed-form states and outputs for one (sequence, head).

    q, k: [T, d_k]; v: [T, d_v]; alpha: [T] or [T, d_k]; beta: [T];
    S0: [d_v, d_k].  Returns (o [T, d_v], [S_1, ..., S_T]).
    """
    T, dk = k.shape
    A = [transition(k[t], alpha[t], beta[t]) for t in range(T)]
    I = _eye(dk, k)
    states, outs = [], []
    for t in range(T):
        # Phi(a, t) = A_a ... A_t  (tokens a..t inclusive, 0-based)
        def phi(a):
            P = I.copy()
            for s in range(a, t + 1):
                P = P.dot(A[s])
            return P
        S = S0.dot(phi(0))
        for tau in range(t + 1):
            S = S + (beta[tau] * np.outer(v[tau], k[tau])).dot(phi(tau + 1))
        states.append(S)
        outs.append(S.dot(q[t]))
    return np.array(outs), states
