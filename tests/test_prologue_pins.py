"""Pins for the prologue oracle (short causal convolution with its state,
q/k L2 normalisation, gate and beta maps).  Each check compares the oracle with
something other than its own formula: a library filter routine, the impulse
response the definition fixes, invariants (unit norm, split invariance, state
pass-through) and library special functions.  The convolution's kernel size
comes from the page "Qwen3.8-Flash-Next and GLM-5.3-Flash share a 3:1
long-context pattern" (section "Kimi Delta Attention extends recurrent memory
control"); the state handed from prefill to decode from the page "How the New
Flash Models Work: Inside GLM-5.3-Flash and Qwen3.8-Flash-Next" (section
"Serving: prefill and decode are different problems").
"""
import numpy as np
import pytest
from scipy import signal, special

from oracle import prologue as P


def _rng(seed):
    return np.random.default_rng(seed)


def test_conv_matches_library_fir_filter_from_zero_state():
    r = _rng(1)
    x = r.standard_normal((37, 5))
    w = r.standard_normal((5, 4))
    y, _ = P.causal_conv(x, w)
    for c in range(5):
        # lfilter: y[n] = sum_k b[k] x[n-k]; the current token takes w[:, 3]
        ref = signal.lfilter(w[c, ::-1], [1.0], x[:, c])
        np.testing.assert_allclose(y[:, c], ref, rtol=1e-13, atol=1e-13)


def test_conv_matches_library_fir_filter_with_state():
    r = _rng(2)
    x = r.standard_normal((20, 3))
    w = r.standard_normal((3, 4))
    s = r.standard_normal((1, 3, 3))
    y, s_out = P.causal_conv(x, w, s)
    for c in range(3):
        u = np.concatenate([s[0, c], x[:, c]])    # the three earlier inputs, oldest first
        ref = signal.lfilter(w[c, ::-1], [1.0], u)[3:]
        np.testing.assert_allclose(y[:, c], ref, rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(s_out[0], x[-3:].T)


def test_impulse_response_is_the_taps_in_time_order():
    w = np.array([[0.5, -2.0, 3.0, 7.0]])
    x = np.zeros((6, 1))
    x[0, 0] = 1.0
    y, _ = P.causal_conv(x, w)
    # token t sees the impulse t steps back, i.e. through tap 3 - t
    np.testing.assert_array_equal(y[:, 0], [7.0, 3.0, -2.0, 0.5, 0.0, 0.0])


def test_identity_taps_pass_inputs_through():
    r = _rng(3)
    x = r.standard_normal((9, 4))
    w = np.tile([0.0, 0.0, 0.0, 1.0], (4, 1))
    y, s = P.causal_conv(x, w, r.standard_normal((1, 4, 3)))
    np.testing.assert_array_equal(y, x)
    np.testing.assert_array_equal(s[0], x[-3:].T)


def test_state_never_leaks_across_sequences():
    r = _rng(4)
    x = r.standard_normal((12, 2))
    w = r.standard_normal((2, 4))
    cu = [0, 5, 12]
    y, _ = P.causal_conv(x, w, None, cu)
    y0, _ = P.causal_conv(x[:5], w)
    y1, _ = P.causal_conv(x[5:], w)
    np.testing.assert_array_equal(y, np.concatenate([y0, y1]))


def test_split_at_any_token_with_state_handoff_is_exact():
    r = _rng(5)
    x = r.standard_normal((15, 3))
    w = r.standard_normal((3, 4))
    s0 = r.standard_normal((1, 3, 3))
    y, s = P.causal_conv(x, w, s0)
    for cut in (1, 2, 3, 7, 14):
        ya, sa = P.causal_conv(x[:cut], w, s0)
        yb, sb = P.causal_conv(x[cut:], w, sa)
        np.testing.assert_array_equal(np.concatenate([ya, yb]), y)
        np.testing.assert_array_equal(sb, s)


@pytest.mark.parametrize("L", [0, 1, 2])
def test_short_and_empty_sequences_shift_the_state(L):
    r = _rng(6 + L)
    s0 = r.standard_normal((1, 2, 3))
    x = r.standard_normal((L, 2))
    _, s = P.causal_conv(x, r.standard_normal((2, 4)), s0)
    expect = np.concatenate([s0[0], x.T], axis=1)[:, -3:]
    np.testing.assert_array_equal(s[0], expect)


def test_normalised_heads_have_unit_norm_and_keep_direction():
    r = _rng(7)
    y = r.standard_normal((6, 3 * 16)) * 5.0
    z = P.l2_normalise(y, 16).reshape(6, 3, 16)
    n2 = np.sum(y.reshape(6, 3, 16) ** 2, axis=-1)
    np.testing.assert_allclose(np.sum(z * z, axis=-1), n2 / (n2 + P.EPS), rtol=1e-14)
    cos = np.sum(z * y.reshape(6, 3, 16), axis=-1) / np.sqrt(n2 * np.sum(z * z, axis=-1))
    np.testing.assert_allclose(cos, 1.0, rtol=1e-14)


def test_gate_and_beta_maps_match_library_special_functions():
    x = np.linspace(-30.0, 30.0, 121)
    np.testing.assert_allclose(P.sigmoid(x), special.expit(x), rtol=1e-15, atol=0)
    np.testing.assert_allclose(P.softplus(x), np.log1p(np.exp(x)), rtol=1e-14)
    np.testing.assert_allclose(P.silu(x), x * special.expit(x), rtol=1e-14, atol=1e-300)


def test_gate_range_of_the_workloads():
    # c = 0.05 with x ~ N(0, 1): alpha = exp(g) > 0.9 exactly when x < 1.97 (97.6 %)
    x = _rng(8).standard_normal((1000, 4))
    out = P.prologue(np.zeros((1000, 1, 16)), np.zeros((1000, 1, 16)), np.zeros((1000, 4, 16)),
                     np.zeros((16, 4)), np.zeros((16, 4)), np.zeros((64, 4)), x,
                     np.full(4, 0.05), x)
    a = np.exp(out["g"])
    assert np.all(out["g"] < 0) and np.all(a > 0.8) and abs(np.mean(a > 0.9) - 0.976) < 0.02
    assert np.all((out["beta"] > 0) & (out["beta"] < 1))


def test_prologue_wires_q_k_v_taps_and_state_slices():
    r = _rng(9)
    T, Hqk, H, dk, dv = 7, 1, 2, 4, 8
    xq, xk, xv = r.standard_normal((T, Hqk, dk)), r.standard_normal((T, Hqk, dk)), r.standard_normal((T, H, dv))
    wq, wk, wv = r.standard_normal((dk, 4)), r.standard_normal((dk, 4)), r.standard_normal((H * dv, 4))
    st = r.standard_normal((1, 2 * dk + H * dv, 3))
    out = P.prologue(xq, xk, xv, wq, wk, wv, r.standard_normal((T, H, dk)), np.ones(H),
                     r.standard_normal((T, H)), conv_state=st, use_silu=True, normalize_qk=False)
    for x, w, lo, key in ((xq, wq, 0, "q"), (xk, wk, dk, "k"), (xv, wv, 2 * dk, "v")):
        C = w.shape[0]
        for c in range(C):
            u = np.concatenate([st[0, lo + c], x.reshape(T, -1)[:, c]])
            ref = signal.lfilter(w[c, ::-1], [1.0], u)[3:]
            np.testing.assert_allclose(out[key].reshape(T, -1)[:, c], ref * special.expit(ref),
                                       rtol=1e-12, atol=1e-14)
        np.testing.assert_array_equal(out["conv_state_out"][0, lo:lo + C], x.reshape(T, -1)[-3:].T)
    # per-channel gate: -c_h * softplus broadcast over d_k
    xg = r.standard_normal((T, H, dk))
    out2 = P.prologue(xq, xk, xv, wq, wk, wv, xg, np.array([0.5, 2.0]), np.zeros((T, H)))
    np.testing.assert_allclose(out2["g"][:, 1], -2.0 * np.log1p(np.exp(xg[:, 1])), rtol=1e-14)
