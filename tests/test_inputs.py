"""The seeded input generator: deterministic, thread-count independent, and
producing the value distributions the workloads call for."""
import numpy as np
import torch

from gated_delta_rule_151_b200 import inputs as I


def test_deterministic_and_seed_dependent():
    a = I.make_inputs(total_T=100, H=3, d_k=16, seed=3)
    b = I.make_inputs(total_T=100, H=3, d_k=16, seed=3)
    c = I.make_inputs(total_T=100, H=3, d_k=16, seed=4)
    for x, y in ((a.q, b.q), (a.k, b.k), (a.v, b.v), (a.g, b.g), (a.beta, b.beta)):
        assert torch.equal(x, y)
    assert not torch.equal(a.q, c.q)


def test_thread_count_does_not_change_values(monkeypatch):
    kw = dict(total_T=5000, H=4, d_k=128, seed=1, gate_mode=I.CHANNEL)
    monkeypatch.setattr(I, "_threads", lambda: 1)
    a = I.make_inputs(**kw)
    monkeypatch.setattr(I, "_threads", lambda: 7)
    b = I.make_inputs(**kw)
    assert torch.equal(a.k, b.k) and torch.equal(a.g, b.g)
    assert len(I._blocks((5000, 4, 128))) > 1


def test_distributions():
    x = I.make_inputs(total_T=4096, H=2, d_k=128, seed=0, c=0.05, gate_mode=I.CHANNEL,
                      h0_std=0.02)
    kn = x.k.float().norm(dim=-1)
    assert torch.all((kn - 1).abs() < 2 ** -7)           # bf16-rounded unit vectors
    assert x.q.dtype == torch.bfloat16 and x.g.dtype == torch.float32
    assert torch.all(x.g <= 0) and torch.all(x.beta > 0) and torch.all(x.beta < 1)
    alpha = torch.exp(x.g.double())
    frac_below = float((alpha < 0.9).double().mean())
    assert 0.005 < frac_below < 0.06                     # exp(-softplus(N(0,1)) * 0.05)
    assert abs(float(x.h0.std()) - 0.02) < 1e-3
    assert x.h0.shape == (1, 2, 128, 128)


def test_rounding_is_round_to_nearest_even_via_fp32():
    x = I.make_inputs(total_T=64, H=1, d_k=16, seed=2, io_dtype=torch.float32)
    y = I.make_inputs(total_T=64, H=1, d_k=16, seed=2, io_dtype=torch.bfloat16)
    assert torch.equal(x.v.to(torch.bfloat16), y.v)


def test_varlen_cuts():
    cu = I.random_cu_seqlens(0, 262144, 8)
    assert cu[0] == 0 and cu[-1] == 262144 and len(cu) == 9
    assert np.all(np.diff(cu) > 0)
    assert np.array_equal(cu, I.random_cu_seqlens(0, 262144, 8))


def test_workload_shapes():
    t = I.workload("tiny_gdn")
    assert (t.total_T, t.H, t.d_k, t.d_v, t.num_seqs) == (64, 2, 16, 16, 1)
    assert t.io_dtype == torch.float32 and t.h0 is None and t.g.shape == (64, 2)


def test_decode_view_roundtrip():
    x = torch.arange(3 * 4 * 2).reshape(3 * 4, 2)
    dv = I.decode_view(x, 3)
    assert dv.shape == (4, 3, 2)
    assert torch.equal(dv[1, 2], x[2 * 4 + 1])


def test_prologue_inputs_shapes_and_determinism():
    a = I.make_prologue_inputs(total_T=10, H=4, H_qk=2, d_k=16, d_v=32, cu_seqlens=[0, 3, 3, 10],
                               gate_mode=I.CHANNEL, io_dtype=torch.float32, seed=3)
    b = I.make_prologue_inputs(total_T=10, H=4, H_qk=2, d_k=16, d_v=32, cu_seqlens=[0, 3, 3, 10],
                               gate_mode=I.CHANNEL, io_dtype=torch.float32, seed=3)
    assert a.xq.shape == (10, 2, 16) and a.xv.shape == (10, 4, 32)
    assert a.wq.shape == (32, 4) and a.wv.shape == (128, 4) and a.xg.shape == (10, 4, 16)
    assert a.conv_state.shape == (3, 2 * 32 + 128, 3) and a.num_seqs == 3
    assert torch.equal(a.xq, b.xq) and torch.equal(a.conv_state, b.conv_state)
    assert not torch.equal(a.xq, a.xk)
    p = I.prologue_workload()
    assert p.xq.dtype == torch.bfloat16 and p.total_T == 8192 and p.gscale.shape == (16,)
