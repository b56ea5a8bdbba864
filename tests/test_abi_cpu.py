"""The C ABI library on a machine without a GPU: it loads, exports every
symbol include/gdr.h declares, and rejects invalid arguments on the host
before touching CUDA (no compute call is made here)."""
import ctypes
import os
import re

import pytest
import torch

from gated_delta_rule_151_b200 import gdr

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdr.h")

A = 0x7f0000000000          # a 16-byte aligned fake device address (never dereferenced)
MIS = A + 4                 # misaligned


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GDR_API\s+[\w\s\*]+?\b(gdr_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return gdr.load_library()


def test_header_declares_the_binding_names():
    assert declared_symbols() == sorted(gdr.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(gdr.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(raw, name), name


def test_status_strings(lib):
    for s in range(6):
        assert gdr.gdr_status_string(s).startswith("GDR_")
    assert "UNKNOWN" in gdr.gdr_status_string(99)


def _prefill(lib, **kw):
    args = dict(q=A, k=A, v=A, g=A, beta=A, h0=None, cu=None, N=1, T=64, H=2, dk=16, dv=16,
                gate=0, io=0, o=A, fin=A, ws=None, wsb=0, stream=None)
    args.update(kw)
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.gdr_prefill_chunked(P(args["q"]), P(args["k"]), P(args["v"]), P(args["g"]),
                                   P(args["beta"]), P(args["h0"]), P(args["cu"]), args["N"],
                                   args["T"], args["H"], args["dk"], args["dv"], args["gate"],
                                   args["io"], P(args["o"]), P(args["fin"]), P(args["ws"]),
                                   args["wsb"], args["stream"])


@pytest.mark.parametrize("kw", [
    dict(q=None), dict(k=None), dict(v=None), dict(g=None), dict(beta=None), dict(o=None),
    dict(q=MIS), dict(v=MIS), dict(o=MIS), dict(fin=MIS), dict(h0=MIS), dict(cu=MIS),
    dict(beta=A + 2), dict(g=A + 2), dict(g=A + 4, gate=1),
    dict(dk=48), dict(dv=256), dict(dk=0), dict(H=0), dict(T=-1), dict(N=-1),
    dict(N=3, T=64),              # 64 tokens do not split into 3 equal sequences
    dict(N=0, T=64), dict(gate=2), dict(io=5),
])
def test_prefill_rejects_invalid_arguments(lib, kw):
    assert _prefill(lib, **kw) == gdr.GDR_ERR_INVALID_ARG


def test_scalar_gate_and_beta_need_only_element_alignment(lib):
    # a valid request would launch a kernel, so only the validation outcome is
    # observed: anything but INVALID_ARG means the pointers were accepted
    assert _prefill(lib, N=0, T=0, beta=A + 4, g=A + 4, q=None, k=None, v=None,
                    o=None) == gdr.GDR_OK


def test_prefill_empty_problem_is_a_no_op(lib):
    assert _prefill(lib, N=0, T=0, q=None, k=None, v=None, g=None, beta=None, o=None) == gdr.GDR_OK


def _decode(lib, **kw):
    args = dict(q=A, k=A, v=A, g=A, beta=A, state=A, N=4, H=2, dk=128, dv=128, gate=0, io=1,
                o=A, stream=None)
    args.update(kw)
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.gdr_decode_step(P(args["q"]), P(args["k"]), P(args["v"]), P(args["g"]),
                               P(args["beta"]), P(args["state"]), args["N"], args["H"], args["dk"],
                               args["dv"], args["gate"], args["io"], P(args["o"]), args["stream"])


@pytest.mark.parametrize("kw", [
    dict(q=None), dict(state=None), dict(o=None), dict(state=MIS), dict(k=MIS), dict(dk=100),
    dict(beta=A + 1), dict(g=A + 8, gate=1),
    dict(dv=8), dict(N=-1), dict(H=-2), dict(gate=7), dict(io=3),
])
def test_decode_rejects_invalid_arguments(lib, kw):
    assert _decode(lib, **kw) == gdr.GDR_ERR_INVALID_ARG


def test_decode_empty_batch_is_a_no_op(lib):
    assert _decode(lib, N=0) == gdr.GDR_OK


def test_workspace_and_path_queries(lib):
    assert gdr.gdr_prefill_workspace_size(1, 64, 2, 16, 16, 0, 0) == 0
    assert gdr.gdr_prefill_path(16, 16, 0, gdr.GDR_F32) == gdr.GDR_PATH_SIMT
    assert gdr.gdr_prefill_path(128, 128, 1, gdr.GDR_F32) == gdr.GDR_PATH_SIMT
    with pytest.raises(gdr.GdrError):
        gdr.gdr_prefill_path(12, 16, 0, 0)
    with pytest.raises(gdr.GdrError):
        gdr.gdr_prefill_workspace_size(-1, 64, 2, 16, 16, 0, 0)


def _split_bytes(N, T, H, equal):
    """The chunk-parallel plan's workspace layout: a 256-byte header (error
    word), the chunk numbering (N + 1 int32), the state slots, then one
    window of 98,848-byte records per (global chunk, head)."""
    rec = 98848
    longest = T // N if equal else T
    max_chunks = -(-longest // 64)
    max_total = N * max_chunks if equal else -(-T // 64) + N
    window = min(max_total, (8 << 30) // (H * rec))
    windows = -(-max_total // window)
    by_window = windows > 1 or N * H > 64
    pieces, nseg = 1, 0
    if not by_window:
        pieces, c, size = 0, 0, 12
        while c < max_chunks and pieces < 32:
            c = max_chunks if pieces + 1 == 32 else min(c + size, max_chunks)
            pieces += 1
            size = (size * 13 + 9) // 10
        ns = min(8, (148 // (N * H) + 3) // 2)   # few chains: the segmented scan
        if ns >= 3 and max_chunks >= 2 * ns:
            nseg, pieces = ns, 1
    if by_window:
        state = (windows - 1) * H * 65536
    elif nseg:
        state = N * H * nseg * 3 * 65536   # incoming state, B and M of every segment
    else:
        state = N * H * 65536 if pieces > 1 else 0
    state_off = (256 + (N + 1) * 4 + 255) // 256 * 256
    rec_off = (state_off + state + 1023) // 1024 * 1024
    return rec_off + window * H * rec, windows


def test_plan_selection_and_workspace_sizes(lib):
    """The tcgen05 family runs as two plans: the chunk-parallel one with the
    reported workspace (98,848 bytes of chunk records per chunk and head, in
    windows of at most 8 GiB), the single-kernel one with 16 bytes."""
    S, CH, BF = gdr.GDR_GATE_SCALAR, gdr.GDR_GATE_CHANNEL, gdr.GDR_BF16
    # room for the packed-length plan and the equal-length one
    nb = gdr.gdr_prefill_workspace_size(1, 8192, 16, 128, 128, S, BF)
    assert nb == max(_split_bytes(1, 8192, 16, False)[0], _split_bytes(1, 8192, 16, True)[0])
    assert gdr.gdr_prefill_plan(1, 8192, 16, 128, 128, S, BF, nb) == gdr.GDR_PATH_TCGEN05_SPLIT
    assert gdr.gdr_prefill_plan(1, 8192, 16, 128, 128, CH, BF, nb) == gdr.GDR_PATH_TCGEN05_SPLIT
    assert gdr.gdr_prefill_plan(1, 8192, 16, 128, 128, S, BF, nb - 1) == gdr.GDR_PATH_TCGEN05
    assert gdr.gdr_prefill_plan(1, 8192, 16, 128, 128, S, BF, 16) == gdr.GDR_PATH_TCGEN05
    with pytest.raises(gdr.GdrError):
        gdr.gdr_prefill_plan(1, 8192, 16, 128, 128, S, BF, 8)
    # more than 64 (sequence, head) chains: a window of global chunks
    nb = gdr.gdr_prefill_workspace_size(8, 262144, 16, 128, 128, S, BF)
    assert nb == _split_bytes(8, 262144, 16, False)[0]
    assert _split_bytes(8, 262144, 16, False)[1] == 1
    assert gdr.gdr_prefill_plan(8, 262144, 16, 128, 128, S, BF, nb) == gdr.GDR_PATH_TCGEN05_SPLIT
    # fp32 I/O and other head sizes: the CUDA-core kernel, no workspace
    assert gdr.gdr_prefill_plan(1, 8192, 16, 128, 128, S, gdr.GDR_F32, 0) == gdr.GDR_PATH_SIMT
    assert gdr.gdr_prefill_plan(1, 8192, 16, 64, 64, S, BF, 0) == gdr.GDR_PATH_SIMT
    # 64 heads x 1400 chunks: records beyond 8 GiB -> windows of global chunks
    nb = gdr.gdr_prefill_workspace_size(1, 89600, 64, 128, 128, S, BF)
    assert nb == max(_split_bytes(1, 89600, 64, False)[0], _split_bytes(1, 89600, 64, True)[0])
    assert _split_bytes(1, 89600, 64, True)[1] == 2
    # a tcgen05 problem without any workspace is refused before any launch
    assert _prefill(lib, dk=128, dv=128, io=1) == gdr.GDR_ERR_WORKSPACE


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(4, 2, 16)
    with pytest.raises(ValueError):
        gdr.gdr_prefill_chunked(x, x, x, torch.zeros(4, 2), torch.zeros(4, 2))


def _prefill_gqa(lib, Hqk, H):
    P = ctypes.c_void_p
    return lib.gdr_prefill_chunked_gqa(P(A), P(A), P(A), P(A), P(A), None, None, 1, 64, Hqk, H,
                                       128, 128, 0, 1, P(A), P(A), None, 0, None)


@pytest.mark.parametrize("Hqk,H", [(0, 4), (3, 4), (8, 4), (-1, 2)])
def test_grouped_heads_must_divide(lib, Hqk, H):
    assert _prefill_gqa(lib, Hqk, H) == gdr.GDR_ERR_INVALID_ARG
    P = ctypes.c_void_p
    st = lib.gdr_decode_step_gqa(P(A), P(A), P(A), P(A), P(A), P(A), 2, Hqk, H, 128, 128, 0, 1,
                                 P(A), None)
    assert st == gdr.GDR_ERR_INVALID_ARG


@pytest.mark.parametrize("T,Hqk,H", [(17, 2, 2), (-1, 2, 2), (4, 3, 4), (4, 0, 2)])
def test_decode_multi_rejects_invalid_arguments(lib, T, Hqk, H):
    P = ctypes.c_void_p
    st = lib.gdr_decode_multi(P(A), P(A), P(A), P(A), P(A), P(A), 2, T, Hqk, H, 128, 128, 0, 1,
                              P(A), None, None)
    assert st == gdr.GDR_ERR_INVALID_ARG
    st = lib.gdr_decode_multi(P(A), P(A), P(A), P(A), P(A), P(A), 2, 4, 2, 2, 128, 128, 0, 1,
                              P(A), P(MIS), None)
    assert st == gdr.GDR_ERR_INVALID_ARG     # misaligned snapshot buffer


_PRO_BASE = 1 << 40
_PRO_NAMES = ("xq", "xk", "xv", "wq", "wk", "wv", "xg", "gs", "xb", "sin", "sout", "cu",
              "q", "k", "v", "g", "beta")
_PRO = {n: _PRO_BASE + (i << 30) for i, n in enumerate(_PRO_NAMES)}   # 1 GiB apart


def _prologue(lib, **kw):
    args = dict(_PRO)
    args.update(cu=None, sin=None, sout=None, N=1, T=64, Hqk=2, H=2, dk=16, dv=16, gate=0, io=0,
                flags=2)
    args.update(kw)
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.gdr_prologue(*(P(args[n]) for n in _PRO_NAMES[:12]), args["N"], args["T"],
                            args["Hqk"], args["H"], args["dk"], args["dv"], args["gate"],
                            args["io"], args["flags"], *(P(args[n]) for n in _PRO_NAMES[12:]), None)


@pytest.mark.parametrize("kw", [
    dict(xq=None), dict(xv=None), dict(q=None), dict(wq=None), dict(gs=None), dict(xb=None),
    dict(beta=None), dict(g=None),
    dict(xq=_PRO["xq"] + 2), dict(q=_PRO["q"] + 8), dict(wv=_PRO["wv"] + 4),
    dict(xg=_PRO["xg"] + 2), dict(xg=_PRO["xg"] + 4, gate=1), dict(g=_PRO["g"] + 4, gate=1),
    dict(sin=_PRO["sin"] + 2), dict(sout=_PRO["sout"] + 1),
    dict(dk=48), dict(dv=256), dict(H=0), dict(Hqk=3), dict(N=0), dict(T=-1),
    dict(N=3, T=64), dict(gate=2), dict(io=5), dict(flags=4),
    # outputs overlapping inputs or each other
    dict(q=_PRO["xq"]), dict(v=_PRO["xv"] + 64), dict(g=_PRO["xg"]), dict(beta=_PRO["xb"]),
    dict(sin=_PRO["sin"], sout=_PRO["sin"] + 12), dict(k=_PRO["q"] + 16),
    dict(sout=_PRO["wq"]),
])
def test_prologue_rejects_invalid_arguments(lib, kw):
    assert _prologue(lib, **kw) == gdr.GDR_ERR_INVALID_ARG


def test_prologue_empty_problem_is_a_no_op(lib):
    assert _prologue(lib, T=0, xq=None, xk=None, xv=None, q=None, k=None, v=None, xg=None,
                     g=None, xb=None, beta=None) == gdr.GDR_OK


_FU_NAMES = ("xq", "xk", "xv", "wq", "wk", "wv", "xg", "gs", "xb", "sin", "sout", "h0", "cu",
             "o", "fin", "ws")
_FU = {n: _PRO_BASE + ((i + 40) << 30) for i, n in enumerate(_FU_NAMES)}


def _fused(lib, **kw):
    args = dict(_FU)
    args.update(cu=None, sin=None, sout=None, h0=None, N=1, T=64, Hqk=2, H=2, dk=128, dv=128,
                gate=0, io=1, flags=2, wsb=1 << 30)
    args.update(kw)
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.gdr_prefill_fused(*(P(args[n]) for n in _FU_NAMES[:13]), args["N"], args["T"],
                                 args["Hqk"], args["H"], args["dk"], args["dv"], args["gate"],
                                 args["io"], args["flags"], P(args["o"]), P(args["fin"]),
                                 P(args["ws"]), args["wsb"], None)


@pytest.mark.parametrize("kw", [
    dict(xq=None), dict(xv=None), dict(o=None), dict(wq=None), dict(gs=None), dict(xb=None),
    dict(xg=None), dict(xq=_FU["xq"] + 2), dict(o=_FU["o"] + 8), dict(fin=_FU["fin"] + 4),
    dict(h0=_FU["h0"] + 8), dict(cu=_FU["cu"] + 2), dict(wv=_FU["wv"] + 4),
    dict(xg=_FU["xg"] + 4, gate=1), dict(sout=_FU["sout"] + 1),
    dict(dk=48), dict(H=0), dict(Hqk=3), dict(N=0), dict(T=-1), dict(N=3, T=64), dict(gate=2),
    dict(io=5), dict(flags=4),
    # outputs overlapping inputs or each other
    dict(o=_FU["xv"]), dict(o=_FU["xq"] + 64), dict(h0=_FU["h0"], fin=_FU["h0"] + 64),
    dict(sin=_FU["sin"], sout=_FU["sin"]),
    dict(sout=_FU["o"]), dict(fin=_FU["wq"]),
])
def test_fused_prefill_rejects_invalid_arguments(lib, kw):
    assert _fused(lib, **kw) == gdr.GDR_ERR_INVALID_ARG


@pytest.mark.parametrize("kw", [dict(dk=64, dv=64), dict(io=0)])
def test_fused_prefill_serves_only_the_tensor_core_shape(lib, kw):
    # fp32 I/O or d != 128: run gdr_prologue and gdr_prefill_chunked_gqa instead
    assert _fused(lib, **kw) == gdr.GDR_ERR_UNSUPPORTED


def test_fused_prefill_final_state_may_be_the_initial_state(lib):
    # aliasing passes validation; without a B200 the call then stops at the
    # tensor-core check, before anything is launched
    st = _fused(lib, h0=_FU["h0"], fin=_FU["h0"])
    assert st != gdr.GDR_ERR_INVALID_ARG


_BW_NAMES = ("q", "k", "v", "g", "beta", "h0", "cu", "do", "dsf", "gq", "gk", "gv", "gg", "gb",
             "gh0", "ws")   # gX: the gradient output for X
_BW = {n: _PRO_BASE + ((i + 20) << 30) for i, n in enumerate(_BW_NAMES)}


def _backward(lib, **kw):
    args = dict(_BW)
    args.update(h0=None, cu=None, dsf=None, gh0=None, N=1, T=64, Hqk=2, H=2, dk=16, dv=16,
                gate=0, io=0, wsb=1 << 30)
    args.update(kw)
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.gdr_backward(*(P(args[n]) for n in _BW_NAMES[:7]), args["N"], args["T"],
                            args["Hqk"], args["H"], args["dk"], args["dv"], args["gate"],
                            args["io"], *(P(args[n]) for n in _BW_NAMES[7:]), args["wsb"], None)


@pytest.mark.parametrize("kw", [
    dict(q=None), dict(do=None), dict(gq=None), dict(gv=None), dict(gg=None), dict(gb=None),
    dict(q=_BW["q"] + 2), dict(gq=_BW["gq"] + 4), dict(g=_BW["g"] + 2),
    dict(g=_BW["g"] + 4, gate=1), dict(gh0=_BW["gh0"] + 4), dict(cu=_BW["cu"] + 2),
    dict(dk=48), dict(dv=256), dict(H=0), dict(Hqk=3), dict(N=0), dict(T=-1), dict(N=3),
    dict(gate=2), dict(io=5),
    dict(gq=_BW["q"]), dict(gv=_BW["v"] + 64), dict(gb=_BW["beta"]), dict(gh0=_BW["gq"]),
])
def test_backward_rejects_invalid_arguments(lib, kw):
    assert _backward(lib, **kw) == gdr.GDR_ERR_INVALID_ARG


@pytest.mark.parametrize("kw", [dict(ws=None), dict(wsb=16), dict(ws=_BW["ws"] + 8)])
def test_backward_rejects_a_missing_or_small_workspace(lib, kw):
    assert _backward(lib, **kw) == gdr.GDR_ERR_WORKSPACE


def test_backward_workspace_size(lib):
    # one state checkpoint per 16 tokens of every sequence, plus one per sequence
    assert gdr.gdr_backward_workspace_size(2, 100, 3, 64, 32) == (2 + 7) * 3 * 32 * 64 * 4
    # d_k = d_v = 128: room for the chunked form, one 475,648-byte record per
    # (chunk, head) for up to ceil(T / 64) + N chunks, after 256 bytes of
    # chunk offsets (more than the token loop's checkpoints)
    assert gdr.gdr_backward_workspace_size(1, 8192, 16, 128, 128) == 256 + (128 + 1) * 16 * 475648
    assert 256 + (128 + 1) * 16 * 475648 > (1 + 512) * 16 * 65536


def test_bindings_reject_host_tensors_before_any_call():
    # argument marshalling only: CPU tensors never reach the library
    x = torch.zeros(8, 2, 16)
    with pytest.raises(ValueError, match="CUDA"):
        gdr.gdr_prologue(x, x, x, torch.zeros(32, 4), torch.zeros(32, 4), torch.zeros(32, 4),
                         torch.zeros(8, 2), torch.ones(2), torch.zeros(8, 2))
    with pytest.raises(ValueError, match="CUDA"):
        gdr.gdr_backward(x, x, x, torch.zeros(8, 2), torch.zeros(8, 2), d_o=x)
    xb = torch.zeros(8, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        gdr.gdr_prefill_fused(xb, xb, xb, torch.zeros(256, 4), torch.zeros(256, 4),
                              torch.zeros(256, 4), torch.zeros(8, 2), torch.ones(2),
                              torch.zeros(8, 2))
    with pytest.raises(ValueError, match="CUDA"):
        gdr.gdr_decode_multi(torch.zeros(1, 2, 2, 16), torch.zeros(1, 2, 2, 16),
                             torch.zeros(1, 2, 2, 16), torch.zeros(1, 2, 2), torch.zeros(1, 2, 2),
                             torch.zeros(1, 2, 16, 16))
