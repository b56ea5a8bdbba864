"""The prologue fused into the chunked prefill (gdr_prefill_fused) against the
fp64 oracles composed: the prologue oracle (short causal convolution with
state, optional SiLU, q/k L2 norms, gate and beta maps) gives q, k, v, g and
beta; q, k and v are rounded to bf16, the type the recurrence takes them in;
the recurrence oracle gives o and the final state, compared element by
element at the contract's bf16 tolerances.  Each case also runs the two
launches the fused entry point replaces (gdr_prologue, then
gdr_prefill_chunked_gqa) and checks that both give the same result, and that
the convolution state handed out is the oracle's, bit for bit.

Cases: ragged varlen batches with one-, two- and three-token sequences (the
convolution's window reaches into the incoming state), an empty sequence,
sequences spanning several 64-token chunks with a ragged tail, grouped heads,
both gate modes, with and without SiLU, incoming convolution state and
initial state, and the 8192-token, 16-head GDN shape."""
import numpy as np
import pytest
import torch

from oracle import prologue as P
from gated_delta_rule_151_b200 import gdr
from gated_delta_rule_151_b200 import inputs as I
from _util import TOL_BF16_O, TOL_BF16_STATE_REL, check, oracle_prefill, rel_frob

pytestmark = pytest.mark.gpu


def _h0(seed, N, H):
    rng = np.random.default_rng(np.random.SeedSequence(seed, spawn_key=(77,)))
    return torch.from_numpy((rng.standard_normal((N, H, 128, 128)) * 0.02).astype(np.float32))


def _case(T, H, Hqk, mode, cu, silu, norm, state, h0, seed):
    # without the q/k norms the keys keep the convolution's scale: small taps
    # keep beta |k|^2 below 2, where every token's map is non-expansive (with
    # taps of 0.5, |k|^2 is about 128 and the recurrence itself diverges)
    pi = I.make_prologue_inputs(total_T=T, H=H, H_qk=Hqk, d_k=128, cu_seqlens=cu,
                                num_seqs=1 if cu is not None else 2, gate_mode=mode,
                                io_dtype=torch.bfloat16, c=0.05, tap_std=0.5 if norm else 0.03,
                                state_std=1.0 if state else 0.0, seed=seed)
    N = pi.cu_seqlens.numel() - 1
    init = _h0(seed, N, H) if h0 else None
    return pi, init


def _run_fused(pi, init, use_cu, silu, norm):
    d = lambda x: None if x is None else x.cuda()
    N = pi.cu_seqlens.numel() - 1
    Call = 2 * pi.wq.shape[0] + pi.wv.shape[0]
    st_out = torch.full((N, Call, 3), float("nan"), device="cuda")
    ws = torch.empty(gdr.gdr_prefill_workspace_size(
        N, pi.xq.shape[0], pi.xv.shape[1], 128, 128,
        gdr.GDR_GATE_SCALAR if pi.xg.dim() == 2 else gdr.GDR_GATE_CHANNEL, gdr.GDR_BF16),
        dtype=torch.uint8, device="cuda")
    o, fin = gdr.gdr_prefill_fused(
        d(pi.xq), d(pi.xk), d(pi.xv), d(pi.wq), d(pi.wk), d(pi.wv), d(pi.xg), d(pi.gscale),
        d(pi.xb), d(pi.conv_state), d(init), d(pi.cu_seqlens) if use_cu else None, num_seqs=N,
        conv_state_out=st_out, silu=silu, normalize_qk=norm, workspace=ws)
    torch.cuda.synchronize()
    gdr.gdr_prefill_check_workspace(ws)
    return o, fin, st_out


def _run_two_launches(pi, init, use_cu, silu, norm):
    d = lambda x: None if x is None else x.cuda()
    N = pi.cu_seqlens.numel() - 1
    cu = d(pi.cu_seqlens) if use_cu else None
    Call = 2 * pi.wq.shape[0] + pi.wv.shape[0]
    st_out = torch.full((N, Call, 3), float("nan"), device="cuda")
    q, k, v, g, b = gdr.gdr_prologue(d(pi.xq), d(pi.xk), d(pi.xv), d(pi.wq), d(pi.wk), d(pi.wv),
                                     d(pi.xg), d(pi.gscale), d(pi.xb), d(pi.conv_state), cu,
                                     num_seqs=N, conv_state_out=st_out, silu=silu,
                                     normalize_qk=norm)
    o, fin = gdr.gdr_prefill_chunked_gqa(q, k, v, g, b, d(init), cu, num_seqs=N)
    torch.cuda.synchronize()
    return o, fin, st_out


def _oracle(pi, init, silu, norm):
    ref = P.prologue(pi.xq, pi.xk, pi.xv, pi.wq, pi.wk, pi.wv, pi.xg, pi.gscale, pi.xb,
                     cu_seqlens=pi.cu_seqlens.numpy(), conv_state=pi.conv_state,
                     use_silu=silu, normalize_qk=norm)
    bf = lambda a: torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16)  # noqa: E731
    inp = I.Inputs(q=bf(ref["q"]), k=bf(ref["k"]), v=bf(ref["v"]),
                   g=torch.from_numpy(ref["g"].astype(np.float32)),
                   beta=torch.from_numpy(ref["beta"].astype(np.float32)), h0=init,
                   cu_seqlens=pi.cu_seqlens, gate_mode=pi.gate_mode, io_dtype=torch.bfloat16)
    o_ref, f_ref = oracle_prefill(inp)
    return inp, o_ref, f_ref, ref["conv_state_out"]


CASES = [
    # T, H, H_qk, mode, cu (None: 2 equal sequences), silu, norm, conv state, h0
    (333, 3, 3, I.SCALAR, [0, 1, 3, 6, 71, 200, 333], True, True, True, True),
    (333, 3, 3, I.CHANNEL, [0, 1, 3, 6, 71, 200, 333], True, True, True, True),
    (300, 4, 2, I.SCALAR, [0, 0, 64, 300], False, True, False, False),
    (300, 4, 2, I.CHANNEL, [0, 0, 64, 300], False, True, True, True),
    (512, 2, 1, I.CHANNEL, None, True, True, True, False),
    (200, 2, 2, I.SCALAR, [0, 2, 130, 200], True, False, True, True),
]


@pytest.mark.parametrize("case", CASES, ids=[f"case{i}" for i in range(len(CASES))])
def test_fused_prefill_matches_the_composed_oracles(case):
    T, H, Hqk, mode, cu, silu, norm, state, h0 = case
    pi, init = _case(T, H, Hqk, mode, cu, silu, norm, state, h0, seed=31 + T + H)
    use_cu = cu is not None
    o, fin, st = _run_fused(pi, init, use_cu, silu, norm)
    inp, o_ref, f_ref, st_ref = _oracle(pi, init, silu, norm)
    check(inp, o, fin, o_ref, f_ref, f"fused {case}")
    assert np.array_equal(st.cpu().numpy().astype(np.float64), st_ref)
    # the two launches it replaces give the same result
    o2, fin2, st2 = _run_two_launches(pi, init, use_cu, silu, norm)
    assert torch.equal(st, st2)
    err_o = float((o.float() - o2.float()).abs().max()) if o.numel() else 0.0
    assert err_o <= TOL_BF16_O / 4, err_o
    f, f2 = fin.cpu().numpy(), fin2.cpu().numpy()
    per = max(rel_frob(f[n, h], f2[n, h]) for n in range(f.shape[0]) for h in range(f.shape[1]))
    assert per <= TOL_BF16_STATE_REL / 4, per


def test_fused_prefill_at_the_gdn_prefill_shape():
    """8192 tokens, 16 heads, SiLU and q/k norms, incoming convolution state:
    every element of o and of the final state against the composed oracles."""
    pi, init = _case(8192, 16, 16, I.SCALAR, [0, 8192], True, True, True, False, seed=5)
    o, fin, st = _run_fused(pi, init, True, True, True)
    inp, o_ref, f_ref, st_ref = _oracle(pi, init, True, True)
    check(inp, o, fin, o_ref, f_ref, "fused gdn_prefill shape")
    assert np.array_equal(st.cpu().numpy().astype(np.float64), st_ref)


def test_fused_prefill_without_tokens_passes_the_states_through():
    pi, init = _case(64, 2, 2, I.SCALAR, [0, 64], True, True, True, True, seed=9)
    d = lambda x: None if x is None else x.cuda()
    Call = 2 * pi.wq.shape[0] + pi.wv.shape[0]
    st_out = torch.full((1, Call, 3), float("nan"), device="cuda")
    empty = torch.zeros((0, 2, 128), dtype=torch.bfloat16, device="cuda")
    o, fin = gdr.gdr_prefill_fused(
        empty, empty, empty, d(pi.wq), d(pi.wk), d(pi.wv),
        torch.zeros((0, 2), device="cuda"), d(pi.gscale), torch.zeros((0, 2), device="cuda"),
        d(pi.conv_state), d(init), torch.zeros(2, dtype=torch.int32, device="cuda"),
        conv_state_out=st_out)
    torch.cuda.synchronize()
    assert torch.equal(fin.cpu(), init)
    assert torch.equal(st_out.cpu(), pi.conv_state)
