"""Pins for the backward oracle (gradient of the gated delta rule).  The
oracle's reverse sweep is checked against central finite differences of the
independent fp64 forward loop (the C oracle), entry by entry, for both gate
modes with grouped heads, two packed sequences, an initial state and a
final-state adjoint; and against the closed form of the gate-1, beta-0 case,
where the state never changes.  The forward rule is the one on the page "How
the New Flash Models Work: Inside GLM-5.3-Flash and Qwen3.8-Flash-Next"
(section "Linear attention: a fixed-size memory in place of the cache")."""
import numpy as np
import pytest

import oracle
from oracle import backward as B


def _problem(channel, seed):
    r = np.random.default_rng(seed)
    T, Hqk, H, dk, dv = 6, 1, 2, 4, 3
    cu = np.array([0, 2, 6])
    q = r.standard_normal((T, Hqk, dk))
    k = r.standard_normal((T, Hqk, dk)) * 0.5
    v = r.standard_normal((T, H, dv))
    g = -np.abs(r.standard_normal((T, H, dk) if channel else (T, H))) * 0.3
    beta = 1.0 / (1.0 + np.exp(-r.standard_normal((T, H))))
    h0 = r.standard_normal((2, H, dv, dk)) * 0.3
    dO = r.standard_normal((T, H, dv))
    dSf = r.standard_normal((2, H, dv, dk))
    return dict(q=q, k=k, v=v, g=g, beta=beta, h0=h0), cu, dO, dSf


def _loss(x, cu, dO, dSf, channel):
    o, fin = oracle.run(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], cu,
                        channel_gate=channel, nthreads=1)
    return B.loss(o, fin, dO, dSf)


@pytest.mark.parametrize("channel", [False, True])
def test_gradients_match_finite_differences_of_the_forward_loop(channel):
    x, cu, dO, dSf = _problem(channel, 11 + channel)
    grad = B.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], cu, dO, dSf,
                      channel_gate=channel)
    eps = 1e-6
    names = dict(q="dq", k="dk", v="dv", g="dg", beta="dbeta", h0="dh0")
    for name, gname in names.items():
        num = np.zeros_like(x[name])
        for idx in np.ndindex(x[name].shape):
            xp = {kk: vv.copy() for kk, vv in x.items()}
            xm = {kk: vv.copy() for kk, vv in x.items()}
            xp[name][idx] += eps
            xm[name][idx] -= eps
            num[idx] = (_loss(xp, cu, dO, dSf, channel) - _loss(xm, cu, dO, dSf, channel)) / (2 * eps)
        np.testing.assert_allclose(grad[gname], num, rtol=1e-6, atol=1e-8, err_msg=name)


def test_gate_one_beta_zero_closed_form():
    # alpha = 1 and beta = 0: S_t = S_0 for every t, so o_t = S_0 q_t and
    # dq_t = S_0^T dO_t, dh0 = dS_final + sum_t dO_t q_t^T, dk = dv = 0.
    x, cu, dO, dSf = _problem(False, 21)
    x["g"][:] = 0.0
    x["beta"][:] = 0.0
    grad = B.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], cu, dO, dSf)
    for n, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        for h in range(2):
            S0 = x["h0"][n, h]
            for t in range(a, b):
                np.testing.assert_allclose(grad["dq"][t, 0], sum(
                    x["h0"][n, hh].T @ dO[t, hh] for hh in range(2)), rtol=1e-12)
            expect = dSf[n, h] + sum(np.outer(dO[t, h], x["q"][t, 0]) for t in range(a, b))
            np.testing.assert_allclose(grad["dh0"][n, h], expect, rtol=1e-12)
            del S0
    assert np.all(grad["dk"] == 0) and np.all(grad["dv"] == 0)
