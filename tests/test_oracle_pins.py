"""Pins for the fp64 oracle: it is checked here against things other than
itself -- hand-worked examples, an exact rational expansion of the recurrence
into transition-matrix products, closed forms and invariants that follow from
the update rule on the page "How the New Flash Models Work: Inside
GLM-5.3-Flash and Qwen3.8-Flash-Next" (section "Linear attention: a fixed-size
memory in place of the cache") and from the ungated form on the page
"Qwen3.8-Flash vs GLM-5.3-Flash ..." (section "The 3:1 Blueprint: Recurrent
Delta Rules and 2048-Token Indexing").
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import brute_force

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def one_head(q, k, v, g, beta, S0=None, channel=False):
    """Run the oracle on a single (sequence, head) given [T, d] arrays."""
    T, dk = np.shape(k)
    dv = np.shape(v)[1]
    g = np.asarray(g, dtype=np.float64)
    gg = g.reshape(T, 1, dk) if channel else g.reshape(T, 1)
    h0 = None if S0 is None else np.asarray(S0, dtype=np.float64).reshape(1, 1, dv, dk)
    o, fin = oracle.run(np.reshape(q, (T, 1, dk)), np.reshape(k, (T, 1, dk)),
                        np.reshape(v, (T, 1, dv)), gg, np.reshape(beta, (T, 1)), h0,
                        channel_gate=channel, nthreads=1)
    return o[:, 0], fin[0, 0]


def rand_head(rng, T, dk, dv, channel=False, c=0.3, unit=True):
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk))
    if unit:
        q /= np.linalg.norm(q, axis=1, keepdims=True)
        k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal(T)))
    gs = (T, dk) if channel else (T,)
    g = -np.logaddexp(0, rng.standard_normal(gs)) * c
    S0 = rng.standard_normal((dv, dk)) * 0.3
    return q, k, v, g, beta, S0


# ---------------------------------------------------------------- golden ----

@pytest.mark.parametrize("idx", [0, 1])
def test_hand_worked_examples(idx):
    ex = json.load(open(GOLDEN))["examples"][idx]
    channel = ex["gate_mode"] == "channel"
    g = np.log(np.asarray(ex["alpha"], dtype=np.float64))
    o, S = one_head(ex["q"], ex["k"], ex["v"], g, ex["beta"], ex["S0"], channel)
    np.testing.assert_allclose(o, ex["expect_o"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(S, ex["expect_S"], rtol=0, atol=1e-12)


# ---------------------------------------------------- exact brute force ----

def _frac(a):
    return np.vectorize(Fraction, otypes=[object])(np.asarray(a, dtype=np.float64))


@pytest.mark.parametrize("channel", [False, True])
def test_bit_exact_against_rational_expansion(channel):
    """Dyadic inputs with few bits and gates in {1, 1/2, 1/4}: every product in
    the fp64 loop is exact, so it must equal the rational closed form bit for
    bit."""
    rng = np.random.default_rng(11)
    T, dk, dv = 4, 3, 4
    pick = lambda shape, vals: rng.choice(np.asarray(vals, dtype=np.float64), size=shape)
    q = pick((T, dk), [-1, -0.5, 0, 0.25, 0.5, 1])
    k = pick((T, dk), [-1, -0.5, -0.25, 0, 0.25, 0.5, 1])
    v = pick((T, dv), [-2, -1, -0.5, 0.5, 1, 1.5])
    beta = pick((T,), [0.25, 0.5, 1.0])
    S0 = pick((dv, dk), [-1, -0.5, 0, 0.5, 1])
    alpha = pick((T, dk) if channel else (T,), [1.0, 0.5, 0.25])
    g = np.log(alpha)
    assert np.all(np.exp(g) == alpha)  # exp(log(2^-m)) is exact for these
    o, S = one_head(q, k, v, g, beta, S0, channel)
    eo, states = brute_force.expand(_frac(q), _frac(k), _frac(v), _frac(alpha), _frac(beta), _frac(S0))
    assert np.array_equal(o, eo.astype(np.float64))
    assert np.array_equal(S, states[-1].astype(np.float64))


@pytest.mark.parametrize("channel", [False, True])
def test_rational_expansion_generic_inputs(channel):
    """Generic fp64 inputs, exact rational evaluation of the closed form on
    the very same fp64 values (gates taken as exp(g) in fp64): the loop agrees
    to fp64 rounding."""
    rng = np.random.default_rng(5)
    T, dk, dv = 6, 4, 3
    q, k, v, g, beta, S0 = rand_head(rng, T, dk, dv, channel, c=0.5)
    o, S = one_head(q, k, v, g, beta, S0, channel)
    alpha = np.vectorize(math.exp)(g)
    eo, states = brute_force.expand(_frac(q), _frac(k), _frac(v), _frac(alpha), _frac(beta), _frac(S0))
    np.testing.assert_allclose(o, eo.astype(np.float64), rtol=0, atol=1e-13)
    np.testing.assert_allclose(S, states[-1].astype(np.float64), rtol=0, atol=1e-13)


@pytest.mark.parametrize("channel", [False, True])
def test_float_expansion_d16(channel):
    rng = np.random.default_rng(7)
    T, dk, dv = 8, 16, 16
    q, k, v, g, beta, S0 = rand_head(rng, T, dk, dv, channel)
    o, S = one_head(q, k, v, g, beta, S0, channel)
    eo, states = brute_force.expand(q, k, v, np.exp(g), beta, S0)
    np.testing.assert_allclose(o, eo, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S, states[-1], rtol=0, atol=1e-12)


# ------------------------------------------------------ closed forms ----

def test_zero_write_keeps_state():
    """beta = 0 and gate 1: nothing is erased or written, S_t = S_0 and
    o_t = S_0 q_t."""
    rng = np.random.default_rng(1)
    q, k, v, g, beta, S0 = rand_head(rng, 20, 8, 6)
    o, S = one_head(q, k, v, np.zeros(20), np.zeros(20), S0)
    assert np.array_equal(S, S0)
    np.testing.assert_allclose(o, q @ S0.T, rtol=0, atol=1e-14)


@pytest.mark.parametrize("channel", [False, True])
def test_gate_zero_resets(channel):
    """alpha = 0 (g = -inf) wipes the history: S_t = beta_t v_t k_t^T and
    o_t = beta_t (k_t . q_t) v_t whatever came before."""
    rng = np.random.default_rng(2)
    T, dk, dv = 12, 8, 5
    q, k, v, g, beta, S0 = rand_head(rng, T, dk, dv, channel)
    g = np.full_like(g, -np.inf)
    o, S = one_head(q, k, v, g, beta, S0, channel)
    exp_o = (beta * np.sum(k * q, axis=1))[:, None] * v
    np.testing.assert_allclose(o, exp_o, rtol=0, atol=1e-14)
    np.testing.assert_allclose(S, beta[-1] * np.outer(v[-1], k[-1]), rtol=0, atol=1e-14)


def test_exact_retrieval():
    """Unit key, beta = 1, no decay: (I - k k^T) k = 0, so S_t k_t = v_t."""
    rng = np.random.default_rng(3)
    T, dk, dv = 9, 16, 7
    q, k, v, g, beta, S0 = rand_head(rng, T, dk, dv)
    for t in range(1, T + 1):
        _, S = one_head(q[:t], k[:t], v[:t], np.zeros(t), np.ones(t), S0)
        np.testing.assert_allclose(S @ k[t - 1], v[t - 1], rtol=0, atol=1e-13)


def test_orthonormal_keys_form_outer_product_memory():
    """Orthonormal keys, beta = 1, no decay, S_0 = 0: S_m = sum_i v_i k_i^T,
    the classical linear associative memory, and every pair is retrievable."""
    rng = np.random.default_rng(4)
    dk, dv, m = 12, 6, 9
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm[:, :m].T.copy()
    v = rng.standard_normal((m, dv))
    q = rng.standard_normal((m, dk))
    _, S = one_head(q, k, v, np.zeros(m), np.ones(m), np.zeros((dv, dk)))
    np.testing.assert_allclose(S, v.T @ k, rtol=0, atol=1e-13)
    np.testing.assert_allclose(S @ k.T, v.T, rtol=0, atol=1e-13)


def test_ungated_form_is_lms_step():
    """With D_t = I the rule reads S_t = S_{t-1} + beta_t (v_t - S_{t-1} k_t) k_t^T:
    one Widrow-Hoff (LMS) step on 0.5 ||S k - v||^2.  Evaluated as written."""
    rng = np.random.default_rng(6)
    T, dk, dv = 30, 10, 7
    q, k, v, g, beta, S0 = rand_head(rng, T, dk, dv, unit=False)
    o, S = one_head(q, k, v, np.zeros(T), beta, S0)
    X = S0.copy()
    for t in range(T):
        grad = np.outer(X @ k[t] - v[t], k[t])   # d/dS of 0.5 ||S k - v||^2
        X = X - beta[t] * grad
        np.testing.assert_allclose(o[t], X @ q[t], rtol=0, atol=1e-11)
    np.testing.assert_allclose(S, X, rtol=0, atol=1e-11)


def test_linear_in_initial_state_and_values():
    rng = np.random.default_rng(8)
    T, dk, dv = 15, 8, 8
    for channel in (False, True):
        q, k, v, g, beta, S0 = rand_head(rng, T, dk, dv, channel)
        o_full, S_full = one_head(q, k, v, g, beta, S0, channel)
        o_s, S_s = one_head(q, k, np.zeros_like(v), g, beta, S0, channel)
        o_v, S_v = one_head(q, k, v, g, beta, np.zeros_like(S0), channel)
        np.testing.assert_allclose(o_full, o_s + o_v, rtol=0, atol=1e-13)
        np.testing.assert_allclose(S_full, S_s + S_v, rtol=0, atol=1e-13)
        o3, S3 = one_head(q, k, 3 * v, g, beta, 3 * S0, channel)
        np.testing.assert_allclose(o3, 3 * o_full, rtol=0, atol=1e-12)
        np.testing.assert_allclose(S3, 3 * S_full, rtol=0, atol=1e-12)


def test_uniform_channel_gate_equals_scalar_gate():
    """Kimi Delta Attention is Gated DeltaNet with a per-channel gate: giving
    every key channel the same gate must reproduce the scalar-gate result."""
    rng = np.random.default_rng(9)
    T, dk, dv = 40, 16, 12
    q, k, v, g, beta, S0 = rand_head(rng, T, dk, dv)
    o1, S1 = one_head(q, k, v, g, beta, S0, channel=False)
    o2, S2 = one_head(q, k, v, np.repeat(g[:, None], dk, axis=1), beta, S0, channel=True)
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)


def test_channel_gate_acts_on_key_channels():
    """Gating only key channel j scales column j of S (not row j)."""
    dk = dv = 4
    S0 = np.arange(16, dtype=np.float64).reshape(dv, dk) + 1
    g = np.zeros((1, dk))
    g[0, 2] = np.log(0.5)
    k = np.zeros((1, dk))
    _, S = one_head(np.zeros((1, dk)), k, np.zeros((1, dv)), g, np.zeros(1), S0, channel=True)
    want = S0.copy()
    want[:, 2] *= 0.5
    np.testing.assert_allclose(S, want, rtol=0, atol=1e-15)


def test_householder_reflection_preserves_norm_and_projector_is_idempotent():
    rng = np.random.default_rng(10)
    T, dk, dv = 25, 8, 6
    q, k, v, g, beta, S0 = rand_head(rng, T, dk, dv)
    _, S = one_head(q, k, np.zeros_like(v), np.zeros(T), np.full(T, 2.0), S0)
    assert abs(np.linalg.norm(S) - np.linalg.norm(S0)) < 1e-12
    # beta = 1 with the same key twice: the second erase finds nothing to erase
    kk = np.repeat(k[:1], 2, axis=0)
    _, S1 = one_head(q[:1], kk[:1], np.zeros((1, dv)), np.zeros(1), np.ones(1), S0)
    _, S2 = one_head(q[:2], kk, np.zeros((2, dv)), np.zeros(2), np.ones(2), S0)
    np.testing.assert_allclose(S1, S2, rtol=0, atol=1e-14)


# ------------------------------------------------- packing and handoff ----

def _packed(rng, lens, H, dk, dv, channel):
    T = sum(lens)
    q = rng.standard_normal((T, H, dk)); q /= np.linalg.norm(q, axis=2, keepdims=True)
    k = rng.standard_normal((T, H, dk)); k /= np.linalg.norm(k, axis=2, keepdims=True)
    v = rng.standard_normal((T, H, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal((T, H))))
    g = -np.logaddexp(0, rng.standard_normal((T, H, dk) if channel else (T, H))) * 0.2
    h0 = rng.standard_normal((len(lens), H, dv, dk)) * 0.1
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    return q, k, v, g, beta, h0, cu


@pytest.mark.parametrize("channel", [False, True])
def test_varlen_packing_equals_separate_runs(channel):
    rng = np.random.default_rng(12)
    lens = [5, 0, 17, 1, 9]
    q, k, v, g, beta, h0, cu = _packed(rng, lens, 3, 8, 6, channel)
    o, fin = oracle.run(q, k, v, g, beta, h0, cu, channel_gate=channel)
    for n in range(len(lens)):
        a, b = cu[n], cu[n + 1]
        o1, f1 = oracle.run(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], h0[n:n + 1],
                            channel_gate=channel)
        assert np.array_equal(o[a:b], o1) and np.array_equal(fin[n], f1[0])
    assert np.array_equal(fin[1], h0[1])  # empty sequence keeps its state


@pytest.mark.parametrize("channel", [False, True])
def test_split_with_state_handoff_equals_one_run(channel):
    rng = np.random.default_rng(13)
    q, k, v, g, beta, h0, cu = _packed(rng, [50], 2, 8, 8, channel)
    o, fin = oracle.run(q, k, v, g, beta, h0, channel_gate=channel)
    T1 = 23
    oa, fa = oracle.run(q[:T1], k[:T1], v[:T1], g[:T1], beta[:T1], h0, channel_gate=channel)
    ob, fb = oracle.run(q[T1:], k[T1:], v[T1:], g[T1:], beta[T1:], fa, channel_gate=channel)
    assert np.array_equal(np.concatenate([oa, ob]), o) and np.array_equal(fb, fin)


def test_threads_do_not_change_results():
    rng = np.random.default_rng(14)
    q, k, v, g, beta, h0, cu = _packed(rng, [7, 30, 11], 4, 16, 8, True)
    a = oracle.run(q, k, v, g, beta, h0, cu, nthreads=1)
    b = oracle.run(q, k, v, g, beta, h0, cu, nthreads=5)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_rejects_bad_arguments():
    z = np.zeros((4, 1, 2))
    with pytest.raises(ValueError):
        oracle.run(z, z, z, np.zeros((4, 1)), np.zeros((4, 1)), None, [0, 3])
    with pytest.raises(ValueError):
        oracle.run(z, z, z, np.zeros((4, 2)), np.zeros((4, 1)))


@pytest.mark.parametrize("channel", [False, True])
def test_grouped_heads_equal_replicated_query_key_heads(channel):
    """Value heads sharing a query/key head give exactly the result of giving
    each value head its own copy of that head (the grouping is an index map,
    not arithmetic)."""
    rng = np.random.default_rng(15)
    T, Hqk, grp, dk, dv = 37, 2, 3, 8, 6
    H = Hqk * grp
    q = rng.standard_normal((T, Hqk, dk)); k = rng.standard_normal((T, Hqk, dk))
    k /= np.linalg.norm(k, axis=2, keepdims=True)
    v = rng.standard_normal((T, H, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal((T, H))))
    g = -np.logaddexp(0, rng.standard_normal((T, H, dk) if channel else (T, H))) * 0.3
    h0 = rng.standard_normal((1, H, dv, dk)) * 0.1
    o1, f1 = oracle.run(q, k, v, g, beta, h0, channel_gate=channel)
    rep = np.arange(H) // grp
    o2, f2 = oracle.run(q[:, rep], k[:, rep], v, g, beta, h0, channel_gate=channel)
    assert np.array_equal(o1, o2) and np.array_equal(f1, f2)
    with pytest.raises(ValueError):
        oracle.run(q[:, :1].repeat(4, axis=1), k[:, :1].repeat(4, axis=1), v, g, beta, h0,
                   channel_gate=channel)   # 4 query/key heads do not divide 6 value heads
