"""Chunked prefill on the GPU against the fp64 oracle, element by element,
at sizes that span several 64-token chunks and a ragged tail, plus the
full-size workloads on sampled (sequence, head) pairs, the edge cases
(empty and one-token sequences, g = -inf, in-place state) and memory-safety
canaries (guard bands, NaN-poisoned outputs)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_151_b200 import gdr
from gated_delta_rule_151_b200 import inputs as I
from _util import PLANS, check, gpu_prefill, oracle_prefill, plan_workspace, to_device, TOL_BF16_O

pytestmark = pytest.mark.gpu


def test_tiny_workload_fp32():
    inp = I.workload("tiny_gdn")
    o, fin = gpu_prefill(inp)
    o_ref, fin_ref = oracle_prefill(inp)
    check(inp, o, fin, o_ref, fin_ref, "tiny_gdn")


@pytest.mark.parametrize("T", [1, 63, 64, 65, 127, 129, 300])
@pytest.mark.parametrize("mode", [I.SCALAR, I.CHANNEL])
@pytest.mark.parametrize("plan", PLANS)
def test_ragged_lengths_bf16_d128(T, mode, plan):
    inp = I.make_inputs(total_T=T, H=3, d_k=128, gate_mode=mode, io_dtype=torch.bfloat16,
                        c=0.1, h0_std=0.02, seed=T)
    o, fin = gpu_prefill(inp, plan=plan)
    o_ref, fin_ref = oracle_prefill(inp)
    check(inp, o, fin, o_ref, fin_ref, f"T={T} {mode}")


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 32), (64, 64), (16, 128), (128, 32), (64, 16)])
@pytest.mark.parametrize("mode", [I.SCALAR, I.CHANNEL])
@pytest.mark.parametrize("io", [torch.float32, torch.bfloat16])
def test_head_dims(dk, dv, mode, io):
    inp = I.make_inputs(total_T=130, H=2, d_k=dk, d_v=dv, gate_mode=mode, io_dtype=io, c=0.2,
                        h0_std=0.05, seed=dk * 7 + dv)
    o, fin = gpu_prefill(inp)
    o_ref, fin_ref = oracle_prefill(inp)
    check(inp, o, fin, o_ref, fin_ref, f"dk={dk} dv={dv} {mode} {io}")


@pytest.mark.parametrize("mode", [I.SCALAR, I.CHANNEL])
@pytest.mark.parametrize("d,io,plan", [(128, torch.bfloat16, "split"), (128, torch.bfloat16, "single"),
                                       (32, torch.float32, "split")])
def test_varlen_with_empty_and_short_sequences(mode, d, io, plan):
    lens = [0, 5, 64, 0, 130, 1, 77]
    cu = np.concatenate([[0], np.cumsum(lens)])
    inp = I.make_inputs(total_T=int(cu[-1]), H=2, d_k=d, cu_seqlens=cu, gate_mode=mode,
                        io_dtype=io, c=0.1, h0_std=0.03, seed=3)
    o, fin = gpu_prefill(inp, plan=plan)
    o_ref, fin_ref = oracle_prefill(inp)
    check(inp, o, fin, o_ref, fin_ref, "varlen")
    # empty sequences hand back their initial state exactly
    for n in (0, 3):
        assert torch.equal(fin[n].cpu(), inp.h0[n])


def test_equal_lengths_without_cu_seqlens():
    inp = I.make_inputs(total_T=3 * 100, H=2, d_k=128, num_seqs=3, io_dtype=torch.bfloat16,
                        h0_std=0.02, seed=8)
    o1, f1 = gpu_prefill(inp, use_cu=True)
    o2, f2 = gpu_prefill(inp, use_cu=False)
    assert torch.equal(o1, o2) and torch.equal(f1, f2)


def test_no_initial_state_means_zeros_and_no_final_state_is_allowed():
    inp = I.make_inputs(total_T=200, H=2, d_k=64, io_dtype=torch.float32, seed=5)
    d = to_device(inp)
    o, fin = gdr.gdr_prefill_chunked(d["q"], d["k"], d["v"], d["g"], d["beta"], None, d["cu"])
    o2, fin2 = gdr.gdr_prefill_chunked(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                       torch.zeros_like(fin), d["cu"])
    o3, none = gdr.gdr_prefill_chunked(d["q"], d["k"], d["v"], d["g"], d["beta"], None, d["cu"],
                                       output_final_state=False)
    torch.cuda.synchronize()
    assert none is None
    assert torch.equal(o, o2) and torch.equal(fin, fin2) and torch.equal(o, o3)


@pytest.mark.parametrize("d,io,plan", [(128, torch.bfloat16, "split"), (128, torch.bfloat16, "single"),
                                       (16, torch.float32, "split")])
def test_in_place_state(d, io, plan):
    inp = I.make_inputs(total_T=150, H=2, d_k=d, num_seqs=1, io_dtype=io, h0_std=0.05, seed=6)
    dv = to_device(inp)
    o_sep, f_sep = gdr.gdr_prefill_chunked(dv["q"], dv["k"], dv["v"], dv["g"], dv["beta"],
                                           dv["h0"], dv["cu"], workspace=plan_workspace(plan))
    state = dv["h0"].clone()
    o_in, f_in = gdr.gdr_prefill_chunked(dv["q"], dv["k"], dv["v"], dv["g"], dv["beta"], state,
                                         dv["cu"], final_state=state, workspace=plan_workspace(plan))
    torch.cuda.synchronize()
    assert f_in.data_ptr() == state.data_ptr()
    assert torch.equal(o_sep, o_in) and torch.equal(f_sep, state)


@pytest.mark.parametrize("mode", [I.SCALAR, I.CHANNEL])
@pytest.mark.parametrize("plan", PLANS)
def test_gate_minus_infinity(mode, plan):
    inp = I.make_inputs(total_T=140, H=2, d_k=128, gate_mode=mode, io_dtype=torch.bfloat16,
                        h0_std=0.05, seed=9)
    g = inp.g.clone()
    g[::17] = -float("inf")       # hard resets inside and across chunks
    inp.g = g
    o, fin = gpu_prefill(inp, plan=plan)
    o_ref, fin_ref = oracle_prefill(inp)
    check(inp, o, fin, o_ref, fin_ref, "g=-inf")


@pytest.mark.parametrize("mode", [I.SCALAR, I.CHANNEL])
@pytest.mark.parametrize("plan", PLANS)
def test_guard_bands_and_poisoned_outputs(mode, plan):
    """Outputs live inside larger buffers whose margins hold a sentinel and
    whose interior starts as NaN: every output element must be written and
    nothing outside may change."""
    inp = I.make_inputs(total_T=197, H=3, d_k=128, gate_mode=mode, io_dtype=torch.bfloat16,
                        cu_seqlens=[0, 61, 61, 197], h0_std=0.02, seed=10)
    d = to_device(inp)
    T, H, D, N = inp.total_T, inp.H, 128, inp.num_seqs
    pad = 4096
    sentinel = 12345.0
    obuf = torch.full((pad + T * H * D + pad,), sentinel, dtype=torch.bfloat16, device="cuda")
    fbuf = torch.full((pad + N * H * D * D + pad,), sentinel, dtype=torch.float32, device="cuda")
    o = obuf[pad:pad + T * H * D].view(T, H, D)
    f = fbuf[pad:pad + N * H * D * D].view(N, H, D, D)
    o.fill_(float("nan"))
    f.fill_(float("nan"))
    gdr.gdr_prefill_chunked(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"], d["cu"], o=o,
                            final_state=f, workspace=plan_workspace(plan))
    torch.cuda.synchronize()
    assert torch.all(obuf[:pad] == sentinel) and torch.all(obuf[-pad:] == sentinel)
    assert torch.all(fbuf[:pad] == sentinel) and torch.all(fbuf[-pad:] == sentinel)
    assert not torch.isnan(o.float()).any() and not torch.isnan(f).any()
    o_ref, fin_ref = oracle_prefill(inp)
    check(inp, o, f, o_ref, fin_ref, "guard")


@pytest.mark.parametrize("mode", [I.SCALAR, I.CHANNEL])
def test_split_prefill_with_state_handoff(mode):
    inp = I.make_inputs(total_T=300, H=2, d_k=128, gate_mode=mode, io_dtype=torch.bfloat16,
                        h0_std=0.02, seed=11)
    d = to_device(inp)
    o_full, f_full = gdr.gdr_prefill_chunked(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"])
    T1 = 131
    oa, fa = gdr.gdr_prefill_chunked(d["q"][:T1].contiguous(), d["k"][:T1].contiguous(),
                                     d["v"][:T1].contiguous(), d["g"][:T1].contiguous(),
                                     d["beta"][:T1].contiguous(), d["h0"])
    ob, fb = gdr.gdr_prefill_chunked(d["q"][T1:].contiguous(), d["k"][T1:].contiguous(),
                                     d["v"][T1:].contiguous(), d["g"][T1:].contiguous(),
                                     d["beta"][T1:].contiguous(), fa)
    torch.cuda.synchronize()
    o_ref, fin_ref = oracle_prefill(inp)
    check(inp, torch.cat([oa, ob]), fb, o_ref, fin_ref, "split")
    check(inp, o_full, f_full, o_ref, fin_ref, "full")


def test_prefill_then_decode_handoff():
    """Prefill the first tokens, hand the state to the decode step for the
    rest: the same outputs as the oracle's single pass."""
    T, T1 = 80, 70
    inp = I.make_inputs(total_T=T, H=2, d_k=128, io_dtype=torch.bfloat16, gate_mode=I.CHANNEL,
                        h0_std=0.02, seed=12)
    d = to_device(inp)
    oa, state = gdr.gdr_prefill_chunked(d["q"][:T1].contiguous(), d["k"][:T1].contiguous(),
                                        d["v"][:T1].contiguous(), d["g"][:T1].contiguous(),
                                        d["beta"][:T1].contiguous(), d["h0"])
    outs = [oa]
    for t in range(T1, T):
        outs.append(gdr.gdr_decode_step(d["q"][t:t + 1], d["k"][t:t + 1], d["v"][t:t + 1],
                                        d["g"][t:t + 1], d["beta"][t:t + 1], state))
    torch.cuda.synchronize()
    o_ref, fin_ref = oracle_prefill(inp)
    check(inp, torch.cat(outs), state, o_ref, fin_ref, "prefill->decode")


# ------------------------------------------------ full-size workloads ----

def _sampled(name, heads, seqs=None, plan="split"):
    inp = I.workload(name)
    o, fin = gpu_prefill(inp, plan=plan)
    o_ref, fin_ref = oracle_prefill(inp, heads=heads, seqs=seqs)
    cu = inp.cu_seqlens.numpy()
    seqs = list(range(inp.num_seqs)) if seqs is None else seqs
    tok = np.concatenate([np.arange(cu[s], cu[s + 1]) for s in seqs])
    o_sel = o[torch.from_numpy(tok).cuda()][:, heads]
    f_sel = fin[seqs][:, heads]
    return check(inp, o_sel, f_sel, o_ref, fin_ref, name)


@pytest.mark.parametrize("plan", PLANS)
def test_full_size_gdn_prefill_sampled(plan):
    _sampled("gdn_prefill", heads=[0, 7, 15], plan=plan)


def test_full_size_kda_prefill_sampled():
    _sampled("kda_prefill", heads=[0, 31], seqs=[0, 1])


def test_full_size_varlen_prefill_sampled():
    _sampled("varlen_gdn", heads=[5])


def test_tensor_core_path_is_used_and_reports_no_timeout():
    """bf16, d = 128, scalar gate runs on the tcgen05 kernel; its workspace
    word (set by a bounded wait that gives up) stays clear."""
    assert gdr.gdr_prefill_path(128, 128, gdr.GDR_GATE_SCALAR, gdr.GDR_BF16) == gdr.GDR_PATH_TCGEN05
    inp = I.make_inputs(total_T=333, H=4, d_k=128, num_seqs=3, cu_seqlens=[0, 100, 101, 333],
                        io_dtype=torch.bfloat16, h0_std=0.02, seed=13)
    d = to_device(inp)
    nb = gdr.gdr_prefill_workspace_size(3, 333, 4, 128, 128, gdr.GDR_GATE_SCALAR, gdr.GDR_BF16)
    assert nb >= 4
    assert gdr.gdr_prefill_plan(3, 333, 4, 128, 128, gdr.GDR_GATE_SCALAR, gdr.GDR_BF16,
                                nb) == gdr.GDR_PATH_TCGEN05_SPLIT
    ws = torch.full((nb,), 0xFF, dtype=torch.uint8, device="cuda")
    o, fin = gdr.gdr_prefill_chunked(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"], d["cu"],
                                     workspace=ws)
    gdr.gdr_prefill_check_workspace(ws)
    o_ref, fin_ref = oracle_prefill(inp)
    check(inp, o, fin, o_ref, fin_ref, "tcgen05")


@pytest.mark.parametrize("c_gate", [0.02, 0.3, 1.5, 6.0])
@pytest.mark.parametrize("plan", PLANS)
def test_channel_gate_decay_strengths(c_gate, plan):
    """Kimi Delta Attention on the tensor-core kernel across decay strengths:
    weak and moderate decays take the fp16 scaled-operand path for the
    intra-chunk products, strong ones push the scaled operands past fp16's
    range and take the exact CUDA-core path; both must match the oracle."""
    assert gdr.gdr_prefill_path(128, 128, gdr.GDR_GATE_CHANNEL, gdr.GDR_BF16) == gdr.GDR_PATH_TCGEN05
    inp = I.make_inputs(total_T=320, H=2, d_k=128, gate_mode=I.CHANNEL, io_dtype=torch.bfloat16,
                        c=c_gate, h0_std=0.02, seed=31)
    o, fin = gpu_prefill(inp, plan=plan)
    o_ref, fin_ref = oracle_prefill(inp)
    check(inp, o, fin, o_ref, fin_ref, f"kda c={c_gate}")


@pytest.mark.parametrize("mode", [I.SCALAR, I.CHANNEL])
def test_chunk_parallel_plan_in_windows(mode):
    """64 heads x 89,600 tokens: the chunk records exceed the 8 GiB window,
    so the chunk-parallel plan runs in two windows of global chunks with the
    state handed between them through the workspace (a sequence of 1400
    chunks, windows of 1357).  Sampled heads against the oracle, in-place
    state."""
    T, H = 89600, 64
    nb = gdr.gdr_prefill_workspace_size(1, T, H, 128, 128, 0 if mode == I.SCALAR else 1,
                                        gdr.GDR_BF16)
    assert (1 << 30) < nb < 1400 * H * 98848   # the workspace holds one window, not all records
    inp = I.make_inputs(total_T=T, H=H, d_k=128, gate_mode=mode, io_dtype=torch.bfloat16,
                        c=0.1, h0_std=0.02, seed=51)
    d = to_device(inp)
    state = d["h0"].clone()
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    o, fin = gdr.gdr_prefill_chunked(d["q"], d["k"], d["v"], d["g"], d["beta"], state, d["cu"],
                                     final_state=state, workspace=ws)
    gdr.gdr_prefill_check_workspace(ws)
    heads = [0, 37, 63]
    o_ref, fin_ref = oracle_prefill(inp, heads=heads)
    check(inp, o[:, heads], fin[:, heads], o_ref, fin_ref, "windows")


@pytest.mark.parametrize("mode", [I.SCALAR, I.CHANNEL])
def test_plans_agree(mode):
    """Both tcgen05 plans compute the same chunk algebra (the chunk-parallel
    plan with more of its operands split into high and low halves): their
    outputs agree within the contract tolerances."""
    inp = I.make_inputs(total_T=1000, H=4, d_k=128, gate_mode=mode, io_dtype=torch.bfloat16,
                        cu_seqlens=[0, 333, 334, 1000], c=0.1, h0_std=0.02, seed=52)
    o1, f1 = gpu_prefill(inp, plan="split")
    o2, f2 = gpu_prefill(inp, plan="single")
    assert float((o1.float() - o2.float()).abs().max()) <= TOL_BF16_O
    assert float((f1 - f2).norm() / f2.norm()) <= 1e-3


@pytest.mark.parametrize("mode", [I.SCALAR, I.CHANNEL])
def test_chunk_parallel_plan_in_pipelined_pieces(mode):
    """16 heads x 3 sequences (48 chains, too many for the segmented scan):
    the records of up to 100 chunks per sequence fit one window, which runs as
    pipelined pieces (prep of the next piece beside the chain of this one,
    the state handed between pieces through the workspace).  Sequences of 32
    chunks, one token and 69 chunks, so pieces end inside and after
    sequences.  Sampled heads against the oracle."""
    inp = I.make_inputs(total_T=6400, H=16, d_k=128, gate_mode=mode, io_dtype=torch.bfloat16,
                        cu_seqlens=[0, 2048, 2049, 6400], c=0.1, h0_std=0.02, seed=53)
    nb = gdr.gdr_prefill_workspace_size(3, 6400, 16, 128, 128, 0 if mode == I.SCALAR else 1,
                                        gdr.GDR_BF16)
    assert gdr.gdr_prefill_plan(3, 6400, 16, 128, 128, 0 if mode == I.SCALAR else 1, gdr.GDR_BF16,
                                nb) == gdr.GDR_PATH_TCGEN05_SPLIT
    o, fin = gpu_prefill(inp)
    heads = [0, 9, 15]
    o_ref, fin_ref = oracle_prefill(inp, heads=heads)
    check(inp, o[:, heads], fin[:, heads], o_ref, fin_ref, "pieces")


@pytest.mark.parametrize("mode", [I.SCALAR, I.CHANNEL])
def test_equal_lengths_plan_knows_each_sequence_length(mode):
    # 2 x 6000 tokens x 32 heads: with cu_seqlens the plan bounds a sequence
    # by all 12000 tokens (188 chunks, pipelined pieces past the second
    # sequence's end); without it each sequence has 94 chunks.  Both match
    # the oracle, and the two runs agree.
    inp = I.make_inputs(total_T=12000, H=32, d_k=128, num_seqs=2, gate_mode=mode,
                        io_dtype=torch.bfloat16, c=0.05, h0_std=0.02, seed=90)
    o1, f1 = gpu_prefill(inp, use_cu=True)
    o2, f2 = gpu_prefill(inp, use_cu=False)
    o_ref, fin_ref = oracle_prefill(inp)
    check(inp, o1, f1, o_ref, fin_ref, "with cu_seqlens")
    check(inp, o2, f2, o_ref, fin_ref, "equal lengths")
    assert float((o1.float() - o2.float()).abs().max()) <= 2e-2


@pytest.mark.parametrize("mode", [I.SCALAR, I.CHANNEL])
def test_many_chains_run_by_windows_with_empty_sequences(mode):
    """40 sequences x 2 heads (more than 64 chains): the chunk-parallel plan
    numbers every sequence's chunks on the device and runs the prep kernel
    over the window of global chunks, then one chain CTA per (sequence, head).
    Empty, one-token and multi-chunk sequences, against the oracle."""
    rng = np.random.default_rng(np.random.SeedSequence(71, spawn_key=(99,)))
    lens = rng.choice([0, 1, 5, 63, 64, 65, 130, 200], size=40)
    cu = np.concatenate([[0], np.cumsum(lens)])
    inp = I.make_inputs(total_T=int(cu[-1]), H=2, d_k=128, cu_seqlens=cu, gate_mode=mode,
                        io_dtype=torch.bfloat16, c=0.1, h0_std=0.02, seed=71)
    nb = gdr.gdr_prefill_workspace_size(40, int(cu[-1]), 2, 128, 128,
                                        0 if mode == I.SCALAR else 1, gdr.GDR_BF16)
    assert gdr.gdr_prefill_plan(40, int(cu[-1]), 2, 128, 128, 0 if mode == I.SCALAR else 1,
                                gdr.GDR_BF16, nb) == gdr.GDR_PATH_TCGEN05_SPLIT
    o, fin = gpu_prefill(inp)
    o_ref, fin_ref = oracle_prefill(inp)
    check(inp, o, fin, o_ref, fin_ref, "windows, many chains")
    for n in np.nonzero(lens == 0)[0]:
        assert torch.equal(fin[n].cpu(), inp.h0[n])



@pytest.mark.parametrize("mode", [I.SCALAR, I.CHANNEL])
@pytest.mark.parametrize("case", ["equal", "varlen", "ungated", "strong decay"])
def test_segmented_scan(mode, case):
    """Few chains (here 2 heads): each sequence is cut into 8 segments; the
    segments run from a zero state and their transitions from the identity
    in parallel, the incoming states are composed segment by segment, and the
    segments run again from their true incoming states with outputs.  Segment
    boundaries fall inside chunks' sequences and, with cu_seqlens, sequences
    end inside segments; the ungated rule (the transitions carry the state
    undecayed) and strong decays (transitions near zero) are the extremes."""
    c, cu, T = 0.1, None, 4000
    if case == "varlen":
        cu = [0, 1000, 1001, 2500, 4000]
    inp = I.make_inputs(total_T=T, H=2, d_k=128, gate_mode=mode, io_dtype=torch.bfloat16,
                        cu_seqlens=cu, num_seqs=1, c=(3.0 if case == "strong decay" else c),
                        h0_std=0.05, seed=81)
    if case == "ungated":
        inp.g = torch.zeros_like(inp.g)
    o, fin = gpu_prefill(inp, use_cu=cu is not None)
    o_ref, fin_ref = oracle_prefill(inp)
    check(inp, o, fin, o_ref, fin_ref, f"segments {case} {mode}")


@pytest.mark.parametrize("mode", [I.SCALAR, I.CHANNEL])
def test_three_segments(mode):
    """40 chains (2 sequences x 20 heads): four segments no longer fit the
    SMs in the first phase, three do (40 x 3 = 120 CTAs): segment 0 from the
    initial state, the middle segment from zero and from the identity, one
    composition step, then the middle and last segments from their incoming
    states.  A ragged tail and unequal lengths put the segment boundaries at
    different chunks for the two sequences."""
    inp = I.make_inputs(total_T=1500, H=20, d_k=128, gate_mode=mode, io_dtype=torch.bfloat16,
                        cu_seqlens=[0, 1100, 1500], c=0.1, h0_std=0.05, seed=83)
    nb = gdr.gdr_prefill_workspace_size(2, 1500, 20, 128, 128,
                                        gdr.GDR_GATE_SCALAR if mode == I.SCALAR else gdr.GDR_GATE_CHANNEL,
                                        gdr.GDR_BF16)
    assert gdr.gdr_prefill_plan(2, 1500, 20, 128, 128,
                                gdr.GDR_GATE_SCALAR if mode == I.SCALAR else gdr.GDR_GATE_CHANNEL,
                                gdr.GDR_BF16, nb) == gdr.GDR_PATH_TCGEN05_SPLIT
    o, fin = gpu_prefill(inp)
    o_ref, fin_ref = oracle_prefill(inp)
    check(inp, o, fin, o_ref, fin_ref, f"three segments {mode}")
