"""The chunk algebra of the chunked gradient, restated in fp64 numpy and
checked against the token-loop backward oracle (CPU only; the CUDA kernels
are checked against the same oracle in test_backward_gpu.py).

The chunked form rearranges the gradient of the recurrence per chunk of C
tokens (page "How the New Flash Models Work: Inside GLM-5.3-Flash and
Qwen3.8-Flash-Next", section "Linear attention: a fixed-size memory in place
of the cache", Gated DeltaNet equation, run backwards).  With S the state
entering a chunk, G the within-chunk cumulative log-gate, gamma = e^G,
R_ij = e^{G_i - G_j}:

  forward:  A = strictly-lower(diag(beta) (K K^T) o R), T = (I + A)^-1,
            W = T diag(beta gamma) K, U~ = T diag(beta) V, U = U~ - W S^T,
            S' = e^{G_C} S + U^T K^ with K^_j = k_j e^{G_C - G_j}
  reverse:  with L' the adjoint of S', Y = dO^T diag(gamma) Q and
            Z = P^T dO (P = causal((Q K^T) o R)):
            dU = Z + K^ L'^T,  L = e^{G_C} L' + Y - dU^T W
  local:    dK^ = U L', dW = -dU S, d(gamma Q) = dO S, dP = causal(dO U^T),
            dT = dU (beta V)^T + dW (beta gamma K)^T,
            dA = strictly-lower(-T^T dT T^T),
            and the per-token adjoints of G (reverse-summed into dg).

This is the algebra the chunk prep, the two chains and the chunk-local
kernel compute; a wrong sign, a dropped decay factor or a transposed product
in it fails here against the oracle, which it matches to fp64 rounding."""
import numpy as np
import pytest

from oracle import backward as OB

LOG_GATE_MIN = -20.0


def chunked_gradient(q, k, v, g, beta, h0, dO, dSf, C):
    """One (sequence, head): q, k [T, dk], v, dO [T, dv], g, beta [T],
    h0, dSf [dv, dk]; every chunk of C tokens (the last one ragged)."""
    T = q.shape[0]
    g = np.maximum(g, LOG_GATE_MIN)
    n_chunks = (T + C - 1) // C
    chunks, S = [], h0.copy()
    for c in range(n_chunks):                       # prep and the forward chain
        a, b = c * C, min(T, c * C + C)
        K, Q, V, bt = k[a:b], q[a:b], v[a:b], beta[a:b]
        G = np.cumsum(g[a:b])
        gam, GC = np.exp(G), G[-1]
        R = np.exp(G[:, None] - G[None, :])
        A = np.tril(bt[:, None] * (K @ K.T) * R, -1)
        Tm = np.linalg.inv(np.eye(b - a) + A)
        W = Tm @ (bt[:, None] * gam[:, None] * K)
        Ut = Tm @ (bt[:, None] * V)
        Kh = K * np.exp(GC - G)[:, None]
        P = np.tril((Q @ K.T) * R)
        U = Ut - W @ S.T
        z = dict(a=a, b=b, K=K, Q=Q, V=V, bt=bt, G=G, gam=gam, GC=GC, R=R, A=A, T=Tm, W=W,
                 Kh=Kh, P=P, U=U, S=S.copy(),
                 Y=dO[a:b].T @ (gam[:, None] * Q), Z=P.T @ dO[a:b])
        chunks.append(z)
        S = np.exp(GC) * S + U.T @ Kh
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dg, db = np.zeros(T), np.zeros(T)
    Lam = dSf.copy()
    for z in reversed(chunks):                      # the reverse chain and the local gradients
        a, b = z["a"], z["b"]
        K, Q, V, bt, gam, GC, R, Tm = z["K"], z["Q"], z["V"], z["bt"], z["gam"], z["GC"], z["R"], z["T"]
        dOc, S, U, W, Kh, P = dO[a:b], z["S"], z["U"], z["W"], z["Kh"], z["P"]
        dU = z["Z"] + Kh @ Lam.T
        # local
        dKh = U @ Lam
        dW = -dU @ S
        dQt = dOc @ S
        dP = np.tril(dOc @ U.T)
        dT = dU @ (bt[:, None] * V).T + dW @ (bt[:, None] * gam[:, None] * K).T
        dA = np.tril(-Tm.T @ dT @ Tm.T, -1)
        X1, X2 = Tm.T @ dU, Tm.T @ dW
        dG = np.zeros(b - a)
        dq[a:b] += gam[:, None] * dQt
        dG += gam * np.sum(Q * dQt, 1)
        dv[a:b] += bt[:, None] * X1
        db[a:b] += np.sum(V * X1, 1) + gam * np.sum(K * X2, 1)
        dk[a:b] += (bt * gam)[:, None] * X2
        dG += bt * gam * np.sum(K * X2, 1)
        db[a:b] += np.sum(dA * (K @ K.T) * R, 1)
        M = dA * bt[:, None] * R
        dk[a:b] += (M + M.T) @ K
        E = dA * z["A"] + dP * P
        dG += E.sum(1) - E.sum(0)
        MP = dP * R
        dq[a:b] += MP @ K
        dk[a:b] += MP.T @ Q
        dk[a:b] += np.exp(GC - z["G"])[:, None] * dKh
        dG -= np.sum(Kh * dKh, 1)
        dG[-1] += np.exp(GC) * np.sum(S * Lam) + np.sum(Kh * dKh)
        dg[a:b] = np.cumsum(dG[::-1])[::-1]
        # the adjoint of the state entering the chunk
        Lam = np.exp(GC) * Lam + z["Y"] - dU.T @ W
    dg = np.where(np.asarray(g) > LOG_GATE_MIN, dg, 0.0)
    return dict(dq=dq, dk=dk, dv=dv, dg=dg, dbeta=db, dh0=Lam)


def _case(seed, T, dk, dv, gate_scale, clamp_token=None):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, dk))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((T, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    g = -np.log1p(np.exp(rng.standard_normal(T))) * gate_scale
    if clamp_token is not None:
        g[clamp_token] = -25.0                      # below the clamp: its dg is 0
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(T)))
    h0 = rng.standard_normal((dv, dk)) * 0.1
    dO = rng.standard_normal((T, dv))
    dSf = rng.standard_normal((dv, dk))
    return q, k, v, g, beta, h0, dO, dSf


@pytest.mark.parametrize("T, C, dk, dv, gate_scale, clamp", [
    (37, 8, 6, 5, 0.3, None),      # ragged last chunk, d_k != d_v
    (64, 16, 8, 8, 0.1, None),     # whole chunks only
    (5, 8, 4, 4, 1.0, None),       # one partial chunk
    (50, 8, 5, 7, 0.2, 17),        # a clamped gate inside a chunk
    (1, 4, 3, 3, 0.5, None),       # a single token
])
def test_chunk_algebra_matches_the_token_oracle(T, C, dk, dv, gate_scale, clamp):
    q, k, v, g, beta, h0, dO, dSf = _case(7 + T, T, dk, dv, gate_scale, clamp)
    got = chunked_gradient(q, k, v, g, beta, h0, dO, dSf, C)
    ref = OB.backward(q[:, None], k[:, None], v[:, None], g[:, None], beta[:, None],
                      h0[None, None], None, dO[:, None], dSf[None, None])
    for key in ("dq", "dk", "dv", "dg", "dbeta", "dh0"):
        r = np.asarray(ref[key], dtype=np.float64).reshape(got[key].shape)
        scale = max(float(np.max(np.abs(r))), 1e-30)
        # fp64 rounding, amplified where a clamped gate puts e^{+-20} factors
        # into R: about 1e-9 of the largest entry at worst
        assert float(np.max(np.abs(got[key] - r))) <= 1e-8 * scale, key


def test_chunk_size_does_not_change_the_gradient():
    """The chunking is exact algebra: any chunk size gives the same gradient."""
    args = _case(3, 40, 6, 6, 0.3)
    a = chunked_gradient(*args, C=4)
    b = chunked_gradient(*args, C=16)
    for key in a:
        assert np.allclose(a[key], b[key], rtol=1e-10, atol=1e-12), key


def chunked_gradient_channel(q, k, v, g, beta, h0, dO, dSf, C):
    """The same chunk algebra for a gate per key channel (g [T, dk]), the
    decays carried by the key-side operands: with G the within-chunk
    cumulative log-gate per channel, K~ = K o e^G, K- = K o e^-G,
    Q~ = Q o e^G, K^ = K o e^{G_C - G},

      A = strictly-lower(diag(beta) K~ K-^T), P = causal(Q~ K-^T),
      W = T diag(beta) K~, S' = S Diag(e^{G_C}) + U^T K^,
      L = L' Diag(e^{G_C}) + dO^T Q~ - dU^T W,

    and the adjoint of G per channel from each of K~, K-, K^, Q~ and
    e^{G_C}.  (fp64, moderate gates: e^-G stays in range.)"""
    T = q.shape[0]
    n_chunks = (T + C - 1) // C
    chunks, S = [], h0.copy()
    for c in range(n_chunks):
        a, b = c * C, min(T, c * C + C)
        K, Q, V, bt = k[a:b], q[a:b], v[a:b], beta[a:b]
        G = np.cumsum(g[a:b], axis=0)
        GC = G[-1]
        Kt, Km, Qt = K * np.exp(G), K * np.exp(-G), Q * np.exp(G)
        Kh = K * np.exp(GC - G)
        A = np.tril(bt[:, None] * (Kt @ Km.T), -1)
        Tm = np.linalg.inv(np.eye(b - a) + A)
        W = Tm @ (bt[:, None] * Kt)
        Ut = Tm @ (bt[:, None] * V)
        P = np.tril(Qt @ Km.T)
        U = Ut - W @ S.T
        chunks.append(dict(a=a, b=b, K=K, Q=Q, V=V, bt=bt, G=G, GC=GC, Kt=Kt, Km=Km, Qt=Qt,
                           Kh=Kh, A=A, T=Tm, W=W, P=P, U=U, S=S.copy()))
        S = S * np.exp(GC)[None, :] + U.T @ Kh
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dg, db = np.zeros_like(g), np.zeros(T)
    Lam = dSf.copy()
    for z in reversed(chunks):
        a, b = z["a"], z["b"]
        K, Q, V, bt, G, GC, Tm = z["K"], z["Q"], z["V"], z["bt"], z["G"], z["GC"], z["T"]
        Kt, Km, Qt, Kh, W, P, U, S = z["Kt"], z["Km"], z["Qt"], z["Kh"], z["W"], z["P"], z["U"], z["S"]
        dOc = dO[a:b]
        dU = Kh @ Lam.T + P.T @ dOc
        dKh = U @ Lam
        dP = np.tril(dOc @ U.T)
        dQt = dOc @ S
        dW = -dU @ S
        dT = dW @ (bt[:, None] * Kt).T + dU @ (bt[:, None] * V).T
        X1, X2 = Tm.T @ dU, Tm.T @ dW
        dA = np.tril(-Tm.T @ dT @ Tm.T, -1)
        dKt = bt[:, None] * X2 + bt[:, None] * (dA @ Km)
        dKm = dA.T @ (bt[:, None] * Kt) + dP.T @ Qt
        dQt = dQt + dP @ Km
        dv[a:b] += bt[:, None] * X1
        db[a:b] += np.sum(V * X1, 1) + np.sum(Kt * X2, 1) + np.sum(dA * (Kt @ Km.T), 1)
        dk[a:b] += dKt * np.exp(G) + dKm * np.exp(-G) + dKh * np.exp(GC - G)
        dq[a:b] += dQt * np.exp(G)
        dG = dKt * Kt - dKm * Km - dKh * Kh + dQt * Qt
        dG[-1] += np.exp(GC) * np.sum(S * Lam, 0) + np.sum(dKh * Kh, 0)
        dg[a:b] = np.cumsum(dG[::-1], axis=0)[::-1]
        Lam = Lam * np.exp(GC)[None, :] + dOc.T @ Qt - dU.T @ W
    return dict(dq=dq, dk=dk, dv=dv, dg=dg, dbeta=db, dh0=Lam)


@pytest.mark.parametrize("T, C, dk, dv", [(37, 8, 6, 5), (16, 16, 4, 4), (3, 8, 5, 3)])
def test_channel_gate_chunk_algebra_matches_the_token_oracle(T, C, dk, dv):
    q, k, v, _, beta, h0, dO, dSf = _case(11 + T, T, dk, dv, 0.3)
    rng = np.random.default_rng(100 + T)
    g = -np.log1p(np.exp(rng.standard_normal((T, dk)))) * 0.2   # one log-gate per key channel
    got = chunked_gradient_channel(q, k, v, g, beta, h0, dO, dSf, C)
    ref = OB.backward(q[:, None], k[:, None], v[:, None], g[:, None], beta[:, None],
                      h0[None, None], None, dO[:, None], dSf[None, None])
    for key in ("dq", "dk", "dv", "dg", "dbeta", "dh0"):
        r = np.asarray(ref[key], dtype=np.float64).reshape(got[key].shape)
        scale = max(float(np.max(np.abs(r))), 1e-30)
        assert float(np.max(np.abs(got[key] - r))) <= 1e-9 * scale, key
