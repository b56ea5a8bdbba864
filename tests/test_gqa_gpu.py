"""Grouped query/key heads on the GPU (value head h reads query/key head
h // (H // H_qk), the Qwen Gated DeltaNet layout of 16 query-key heads for 48
value heads) against the fp64 oracle, on every kernel path."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_151_b200 import gdr
from gated_delta_rule_151_b200 import inputs as I
from _util import PLANS, TOL_BF16_O, TOL_BF16_STATE_REL, TOL_F32, check, gpu_prefill, oracle_prefill, rel_frob

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode", [I.SCALAR, I.CHANNEL])
@pytest.mark.parametrize("d,io,plan", [(128, torch.bfloat16, "split"), (128, torch.bfloat16, "single"),
                                       (32, torch.float32, "split")])
def test_prefill_grouped_heads(mode, d, io, plan):
    inp = I.make_inputs(total_T=211, H=6, H_qk=2, d_k=d, gate_mode=mode, io_dtype=io,
                        cu_seqlens=[0, 90, 90, 211], c=0.1, h0_std=0.03, seed=41)
    o, fin = gpu_prefill(inp, plan=plan)
    o_ref, fin_ref = oracle_prefill(inp)
    check(inp, o, fin, o_ref, fin_ref, f"gqa {mode} d={d}")


@pytest.mark.parametrize("plan", PLANS)
def test_prefill_grouped_equals_replicated_heads(plan):
    """The kernels' head mapping is an index map: replicating each query/key
    head over its value heads must give bit-identical results."""
    inp = I.make_inputs(total_T=150, H=6, H_qk=3, d_k=128, io_dtype=torch.bfloat16,
                        h0_std=0.02, seed=42)
    o1, f1 = gpu_prefill(inp, plan=plan)
    rep = torch.arange(6) // 2
    inp.q, inp.k = inp.q[:, rep].contiguous(), inp.k[:, rep].contiguous()
    o2, f2 = gpu_prefill(inp, plan=plan)
    assert torch.equal(o1, o2) and torch.equal(f1, f2)


@pytest.mark.parametrize("mode", [I.SCALAR, I.CHANNEL])
@pytest.mark.parametrize("d,io", [(128, torch.bfloat16), (64, torch.float32)])
def test_decode_grouped_heads(mode, d, io):
    steps, N, H, Hqk = 5, 3, 8, 2
    inp = I.make_inputs(total_T=N * steps, H=H, H_qk=Hqk, d_k=d, num_seqs=N, gate_mode=mode,
                        io_dtype=io, c=0.3, h0_std=0.05, seed=43)
    dev = "cuda"
    qs, ks, vs = (I.decode_view(x, N).to(dev) for x in (inp.q, inp.k, inp.v))
    gs, bs = I.decode_view(inp.g, N).to(dev), I.decode_view(inp.beta, N).to(dev)
    state = inp.h0.to(dev).clone()
    outs = [gdr.gdr_decode_step_gqa(qs[t], ks[t], vs[t], gs[t], bs[t], state) for t in range(steps)]
    torch.cuda.synchronize()
    o = torch.stack(outs).float().cpu().numpy()
    o_ref, f_ref = oracle.loop.run_inputs(inp)
    o_ref = o_ref.reshape(N, steps, H, d).transpose(1, 0, 2, 3)
    f = state.cpu().numpy()
    if io == torch.float32:
        assert np.max(np.abs(o - o_ref)) <= TOL_F32 and np.max(np.abs(f - f_ref)) <= TOL_F32
    else:
        assert np.max(np.abs(o - o_ref)) <= TOL_BF16_O
        assert max(rel_frob(f[n, h], f_ref[n, h]) for n in range(N) for h in range(H)) <= TOL_BF16_STATE_REL


def test_full_size_gqa_prefill_sampled():
    """16 query/key heads x 48 value heads, 8192 tokens, in the launch
    configuration the benchmark times; the oracle checks value heads that
    share and that do not share a query/key head."""
    inp = I.workload("gqa_prefill")
    o, fin = gpu_prefill(inp)
    heads = [0, 1, 2, 47]
    o_ref, fin_ref = oracle_prefill(inp, heads=heads)
    check(inp, o[:, heads], fin[:, heads], o_ref, fin_ref, "gqa_prefill")
