"""The pins of the numpy oracles (prologue and backward) must catch plausible
mistakes.  Each case plants one mistake in a private copy of the oracle's
source (never in the real module), loads it as a separate module, and checks
that the pins' independent references -- a library FIR filter and the
impulse response for the prologue, finite differences of the C forward loop
for the backward -- reject it.  CPU only."""
import importlib.util
import os
import sys
import tempfile

import numpy as np
import pytest
from scipy import signal

import oracle
from oracle import backward as B_real
from oracle import prologue as P_real


def _load_mutant(module, old, new, tag):
    src = open(module.__file__).read()
    assert src.count(old) == 1, (tag, old)
    d = tempfile.mkdtemp()
    path = os.path.join(d, f"mutant_{tag}.py")
    open(path, "w").write(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"mutant_{tag}", path)
    mod = importlib.util.module_from_spec(spec)
    sys.modules[spec.name] = mod
    spec.loader.exec_module(mod)
    return mod


PROLOGUE_MUTATIONS = {
    "taps_reversed": ("acc = acc + w[:, i] * u(t - (TAPS - 1) + i)",
                      "acc = acc + w[:, TAPS - 1 - i] * u(t - (TAPS - 1) + i)"),
    "window_off_by_one": ("acc = acc + w[:, i] * u(t - (TAPS - 1) + i)",
                          "acc = acc + w[:, i] * u(t - TAPS + i)"),
    "state_oldest_last": ("return s_in[n, :, tau - a + TAPS - 1]",
                          "return s_in[n, :, a - tau - 1]"),
    "norm_without_sqrt": ("np.sqrt(np.sum(h * h, axis=-1, keepdims=True) + EPS)",
                          "(np.sum(h * h, axis=-1, keepdims=True) + EPS)"),
}


def _prologue_pins_pass(P):
    r = np.random.default_rng(3)
    x = r.standard_normal((12, 3))
    w = r.standard_normal((3, 4))
    s = r.standard_normal((1, 3, 3))
    y, s_out = P.causal_conv(x, w, s)
    for c in range(3):
        ref = signal.lfilter(w[c, ::-1], [1.0], np.concatenate([s[0, c], x[:, c]]))[3:]
        if not np.allclose(y[:, c], ref, rtol=1e-12, atol=1e-12):
            return False
    imp = np.zeros((6, 1))
    imp[0, 0] = 1.0
    yi, _ = P.causal_conv(imp, np.array([[0.5, -2.0, 3.0, 7.0]]))
    if not np.array_equal(yi[:, 0], [7.0, 3.0, -2.0, 0.5, 0.0, 0.0]):
        return False
    z = P.l2_normalise(r.standard_normal((4, 32)) * 3.0, 16).reshape(4, 2, 16)
    return bool(np.allclose(np.sum(z * z, axis=-1), 1.0, atol=1e-6))


def test_real_prologue_oracle_passes_the_pins():
    assert _prologue_pins_pass(P_real)


@pytest.mark.parametrize("tag", sorted(PROLOGUE_MUTATIONS))
def test_prologue_pins_reject_a_planted_mistake(tag):
    old, new = PROLOGUE_MUTATIONS[tag]
    assert not _prologue_pins_pass(_load_mutant(P_real, old, new, "pro_" + tag))


BACKWARD_MUTATIONS = {
    "adjoint_not_decayed": ("dS = dE * a", "dS = dE"),
    "output_term_dropped": ("dS = dS + np.outer(do, qt)", "dS = dS"),
    "dq_from_previous_state": ("out[\"dq\"][t, hq] += St.T @ do", "out[\"dq\"][t, hq] += Sp.T @ do"),
    "erase_term_of_dk_dropped": ("out[\"dk\"][t, hq] += E.T @ dx", "pass"),
    "gate_gradient_without_a": ("out[\"dg\"][t, h] += (dE * Sp).sum() * a",
                                "out[\"dg\"][t, h] += (dE * Sp).sum()"),
    "dbeta_sign_flipped": ("out[\"dbeta\"][t, h] += (v[t, h] - x) @ du",
                           "out[\"dbeta\"][t, h] += (x - v[t, h]) @ du"),
}


def _backward_matches_finite_differences(Bm):
    r = np.random.default_rng(7)
    T, dk, dv = 4, 3, 2
    x = dict(q=r.standard_normal((T, 1, dk)), k=r.standard_normal((T, 1, dk)) * 0.5,
             v=r.standard_normal((T, 1, dv)), g=-np.abs(r.standard_normal((T, 1))) * 0.3,
             beta=1.0 / (1.0 + np.exp(-r.standard_normal((T, 1)))),
             h0=r.standard_normal((1, 1, dv, dk)) * 0.3)
    dO = r.standard_normal((T, 1, dv))
    dSf = r.standard_normal((1, 1, dv, dk))
    cu = np.array([0, T])
    grad = Bm.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], cu, dO, dSf)

    def loss(xx):
        o, fin = oracle.run(xx["q"], xx["k"], xx["v"], xx["g"], xx["beta"], xx["h0"], cu,
                            channel_gate=False, nthreads=1)
        return B_real.loss(o, fin, dO, dSf)

    eps = 1e-6
    for name, gname in dict(q="dq", k="dk", v="dv", g="dg", beta="dbeta", h0="dh0").items():
        for idx in np.ndindex(x[name].shape):
            xp = {kk: vv.copy() for kk, vv in x.items()}
            xm = {kk: vv.copy() for kk, vv in x.items()}
            xp[name][idx] += eps
            xm[name][idx] -= eps
            num = (loss(xp) - loss(xm)) / (2 * eps)
            if not np.isclose(grad[gname][idx], num, rtol=1e-6, atol=1e-8):
                return False
    return True


def test_real_backward_oracle_matches_finite_differences():
    assert _backward_matches_finite_differences(B_real)


@pytest.mark.parametrize("tag", sorted(BACKWARD_MUTATIONS))
def test_backward_pins_reject_a_planted_mistake(tag):
    old, new = BACKWARD_MUTATIONS[tag]
    assert not _backward_matches_finite_differences(_load_mutant(B_real, old, new, "bwd_" + tag))
