"""Decode step on the GPU against the fp64 oracle.  A T-step decode loop must
reproduce the oracle's token loop over the same T tokens (the decode step is
the recurrence applied once)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_151_b200 import gdr
from gated_delta_rule_151_b200 import inputs as I
from _util import TOL_BF16_O, TOL_BF16_STATE_REL, TOL_F32, rel_frob

pytestmark = pytest.mark.gpu


def run_decode_loop(inp, steps):
    """Feed the workload's tokens one step at a time; returns o [steps, N, H, dv]
    and the final state (both on the CPU)."""
    N = inp.num_seqs
    dev = "cuda"
    qs, ks, vs = (I.decode_view(x, N).to(dev) for x in (inp.q, inp.k, inp.v))
    gs, bs = I.decode_view(inp.g, N).to(dev), I.decode_view(inp.beta, N).to(dev)
    if inp.h0 is not None:
        state = inp.h0.to(dev).clone()
    else:
        state = torch.zeros((N, inp.H, inp.d_v, inp.d_k), device=dev)
    outs = []
    for t in range(steps):
        outs.append(gdr.gdr_decode_step(qs[t], ks[t], vs[t], gs[t], bs[t], state))
    torch.cuda.synchronize()
    return torch.stack(outs).float().cpu().numpy(), state.cpu().numpy()


def compare(inp, o, fin, o_ref, fin_ref):
    N, steps = inp.num_seqs, inp.total_T // inp.num_seqs
    # oracle o is sequence-major [N*steps, H, dv] -> [steps, N, H, dv]
    o_ref = o_ref.reshape(N, steps, *o_ref.shape[1:]).transpose(1, 0, 2, 3)
    err = float(np.max(np.abs(o - o_ref)))
    if inp.io_dtype == torch.float32:
        assert err <= TOL_F32, err
        assert float(np.max(np.abs(fin - fin_ref))) <= TOL_F32
    else:
        assert err <= TOL_BF16_O, err
        per = max(rel_frob(fin[n, h], fin_ref[n, h]) for n in range(fin.shape[0])
                  for h in range(fin.shape[1]))
        assert per <= TOL_BF16_STATE_REL, per
    return err


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 32), (128, 128), (128, 16), (16, 128)])
@pytest.mark.parametrize("mode", [I.SCALAR, I.CHANNEL])
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_decode_loop_matches_oracle(dk, dv, mode, io):
    steps, N = 6, 3
    inp = I.make_inputs(total_T=N * steps, H=2, d_k=dk, d_v=dv, num_seqs=N, gate_mode=mode,
                        io_dtype=io, c=0.3, h0_std=0.05, seed=dk + dv)
    o, fin = run_decode_loop(inp, steps)
    o_ref, fin_ref = oracle.loop.run_inputs(inp)
    compare(inp, o, fin, o_ref, fin_ref)


def test_decode_gate_zero_resets_state():
    N, H, d = 2, 3, 128
    inp = I.make_inputs(total_T=N, H=H, d_k=d, num_seqs=N, io_dtype=torch.float32, h0_std=1.0,
                        seed=4)
    g = torch.full((N, H), -float("inf"), device="cuda")
    q, k, v, b = (x.cuda() for x in (inp.q, inp.k, inp.v, inp.beta))
    state = inp.h0.cuda().clone()
    o = gdr.gdr_decode_step(q, k, v, g, b, state)
    want = (b * (k * q).sum(-1)).unsqueeze(-1) * v
    # the kernel clamps g at -20: the history survives scaled by e^-20
    assert torch.allclose(o, want, atol=1e-6, rtol=0)
    assert torch.allclose(state, b[..., None, None] * v[..., :, None] * k[..., None, :],
                          atol=1e-6, rtol=0)


@pytest.mark.parametrize("name", ["decode_gdn", "decode_kda"])
def test_full_size_decode_workload_sampled(name):
    """The full 256 x 32 x 128 x 128 (512 MiB) state, 512 steps, in the launch
    configuration the benchmark times; the oracle checks 16 sequences (all
    heads) at every step and their final states."""
    inp = I.workload(name)
    o, fin = run_decode_loop(inp, I.DECODE_STEPS)
    seqs = list(range(0, inp.num_seqs, inp.num_seqs // 16))
    o_ref, fin_ref = oracle.loop.run_inputs(inp, seqs=seqs)
    N, steps = len(seqs), I.DECODE_STEPS
    o_ref = o_ref.reshape(N, steps, *o_ref.shape[1:]).transpose(1, 0, 2, 3)
    err = float(np.max(np.abs(o[:, seqs] - o_ref)))
    assert err <= TOL_BF16_O, err
    per = max(rel_frob(fin[s, h], fin_ref[i, h]) for i, s in enumerate(seqs)
              for h in range(inp.H))
    assert per <= TOL_BF16_STATE_REL, per
