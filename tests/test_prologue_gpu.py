"""The CUDA prologue (short causal convolution with state, optional SiLU, q/k
L2 normalisation, beta and log-gate maps) against the fp64 prologue oracle,
element by element on the same seeded raw inputs: several 64-token tiles with
ragged, empty and one-token sequences, grouped heads, both gate modes, both
I/O types, one token per sequence (the decode case), and the full
8192-token x 16-head shape.  The convolution state handed out is a copy of
inputs and is compared bit for bit."""
import numpy as np
import pytest
import torch

from oracle import prologue as P
from gated_delta_rule_151_b200 import gdr
from gated_delta_rule_151_b200 import inputs as I

pytestmark = pytest.mark.gpu

# Outputs are computed in fp32 and rounded once to the I/O type: bf16 adds at
# most half an ulp (2^-9 relative) to the fp32 error, which stays below 1e-5
# of the tensor's scale for four-term sums and one rsqrt.
RTOL_BF16, RTOL_F32, ATOL_SCALE = 2.0 ** -8, 1e-5, 1e-5
RTOL_MAPS, ATOL_MAPS = 2e-6, 1e-7      # sigmoid / softplus in fp32 library functions


def _run(inp, silu, norm, with_state=True):
    dev = "cuda"
    d = lambda x: None if x is None else x.to(dev)
    st_in = d(inp.conv_state) if with_state else None
    N = inp.num_seqs
    Call = inp.wq.shape[0] * 2 + inp.wv.shape[0]
    st_out = torch.full((N, Call, 3), float("nan"), device=dev)
    cu = d(inp.cu_seqlens) if not inp.meta.get("equal") else None
    q, k, v, g, b = gdr.gdr_prologue(d(inp.xq), d(inp.xk), d(inp.xv), d(inp.wq), d(inp.wk),
                                     d(inp.wv), d(inp.xg), d(inp.gscale), d(inp.xb), st_in, cu,
                                     num_seqs=N, conv_state_out=st_out, silu=silu,
                                     normalize_qk=norm)
    torch.cuda.synchronize()
    ref = P.prologue(inp.xq, inp.xk, inp.xv, inp.wq, inp.wk, inp.wv, inp.xg, inp.gscale, inp.xb,
                     cu_seqlens=inp.cu_seqlens.numpy(), conv_state=st_in.cpu() if with_state else None,
                     use_silu=silu, normalize_qk=norm)
    return dict(q=q, k=k, v=v, g=g, beta=b, conv_state_out=st_out), ref


def _check(got, ref, io):
    rtol = RTOL_BF16 if io == torch.bfloat16 else RTOL_F32
    for key in ("q", "k", "v"):
        x = got[key].float().cpu().numpy().astype(np.float64)
        r = ref[key]
        atol = ATOL_SCALE * max(float(np.max(np.abs(r))), 1e-30)
        err = np.abs(x - r) - (rtol * np.abs(r) + atol)
        assert np.all(err <= 0), (key, float(np.max(err)))
    for key in ("g", "beta"):
        x = got[key].cpu().numpy().astype(np.float64)
        np.testing.assert_allclose(x, ref[key], rtol=RTOL_MAPS, atol=ATOL_MAPS)
    s = got["conv_state_out"].cpu().numpy().astype(np.float64)
    assert np.array_equal(s, ref["conv_state_out"])


@pytest.mark.parametrize("case", [
    # io, d_k, d_v, H_qk, H, gate, silu, norm, state, cu (None = 3 equal sequences of 50)
    (torch.bfloat16, 128, 128, 4, 4, I.SCALAR, True, True, True, [0, 1, 1, 3, 70, 200, 333]),
    (torch.float32, 16, 32, 1, 2, I.CHANNEL, False, True, False, None),
    (torch.bfloat16, 64, 64, 2, 6, I.CHANNEL, True, False, True, [0, 2, 130, 130, 257]),
    (torch.float32, 32, 128, 2, 2, I.SCALAR, True, True, True, [0, 64, 128, 129, 300]),
    (torch.bfloat16, 16, 16, 3, 3, I.SCALAR, False, False, True, [0, 0, 5, 6, 7, 100]),
])
def test_prologue_matches_oracle(case):
    io, dk, dv, Hqk, H, gate, silu, norm, state, cu = case
    if cu is None:
        inp = I.make_prologue_inputs(total_T=150, H=H, H_qk=Hqk, d_k=dk, d_v=dv, num_seqs=3,
                                     gate_mode=gate, io_dtype=io, c=0.1,
                                     state_std=1.0 if state else 0.0, seed=70,
                                     meta={"equal": True})
    else:
        inp = I.make_prologue_inputs(total_T=cu[-1], H=H, H_qk=Hqk, d_k=dk, d_v=dv,
                                     cu_seqlens=cu, gate_mode=gate, io_dtype=io, c=0.1,
                                     state_std=1.0 if state else 0.0, seed=71)
    got, ref = _run(inp, silu, norm, with_state=state)
    _check(got, ref, io)


def test_prologue_one_token_per_sequence_is_a_decode_step():
    N = 64
    inp = I.make_prologue_inputs(total_T=N, H=8, H_qk=4, d_k=128, d_v=128, num_seqs=N,
                                 gate_mode=I.SCALAR, io_dtype=torch.bfloat16, seed=72,
                                 meta={"equal": True})
    got, ref = _run(inp, True, True)
    _check(got, ref, torch.bfloat16)


def test_prologue_full_size_workload():
    inp = I.prologue_workload(seed=0)
    inp.meta["equal"] = True
    got, ref = _run(inp, True, True)
    _check(got, ref, torch.bfloat16)


def test_prologue_split_with_state_handoff_is_bit_exact():
    inp = I.make_prologue_inputs(total_T=1000, H=4, d_k=128, num_seqs=1, gate_mode=I.SCALAR,
                                 io_dtype=torch.bfloat16, seed=73)
    dev = "cuda"
    d = lambda x: x.to(dev)
    Call = 3 * 4 * 128
    args = (d(inp.wq), d(inp.wk), d(inp.wv))
    s0 = d(inp.conv_state)
    whole_s = torch.empty(1, Call, 3, device=dev)
    whole = gdr.gdr_prologue(d(inp.xq), d(inp.xk), d(inp.xv), *args, d(inp.xg), d(inp.gscale),
                             d(inp.xb), s0, None, conv_state_out=whole_s, silu=True)
    parts, s = [], s0
    for a, b in ((0, 1), (1, 3), (3, 517), (517, 1000)):
        s_next = torch.empty(1, Call, 3, device=dev)
        parts.append(gdr.gdr_prologue(d(inp.xq[a:b]), d(inp.xk[a:b]), d(inp.xv[a:b]), *args,
                                      d(inp.xg[a:b]), d(inp.gscale), d(inp.xb[a:b]), s, None,
                                      conv_state_out=s_next, silu=True))
        s = s_next
    torch.cuda.synchronize()
    for i in range(5):
        assert torch.equal(whole[i], torch.cat([p[i] for p in parts]))
    assert torch.equal(whole_s, s)
