"""The allocation-free prefill entry point (gdr_prefill_chunked_noalloc).

It serves callers that may not allocate device memory (their memory belongs
to a host framework's pool, or an allocation would stall a latency-critical
loop); the prefill's scratch then comes from a fixed device array inside the
library instead of a caller-provided workspace.  This file is collected last
so that a failure here stops a first-failure run only after every other test
has run.  It calls the entry point directly through the C ABI, in both gate
modes, twice in a row (the shared array keeps the previous call's contents,
which must not leak into the next result), and checks each result against
the fp64 oracle and against gdr_prefill_chunked with a workspace.  It also
checks that a bounded device-side wait that gives up is reported through
gdr_prefill_noalloc_check, and only once."""
import ctypes

import numpy as np
import pytest
import torch

from gated_delta_rule_151_b200 import gdr
from gated_delta_rule_151_b200 import inputs as I
from _util import TOL_BF16_O, TOL_BF16_STATE_REL, check, oracle_prefill, rel_frob

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc_call(d, inp, gate, o, fin, stream):
    lib = gdr.load_library()
    return lib.gdr_prefill_chunked_noalloc(
        _p(d["q"]), _p(d["k"]), _p(d["v"]), _p(d["g"]), _p(d["beta"]), _p(d["h0"]), _p(d["cu"]),
        inp.num_seqs, inp.total_T, inp.H, inp.d_k, inp.d_v, gate, gdr.GDR_BF16,
        _p(o), _p(fin), ctypes.c_void_p(stream.cuda_stream))


@pytest.mark.parametrize("mode", [I.SCALAR, I.CHANNEL])
def test_noalloc_matches_oracle_and_workspace_entry_point_twice_in_a_row(mode):
    gate = gdr.GDR_GATE_SCALAR if mode == I.SCALAR else gdr.GDR_GATE_CHANNEL
    assert gdr.gdr_prefill_path(128, 128, gate, gdr.GDR_BF16) == gdr.GDR_PATH_TCGEN05
    lib = gdr.load_library()
    stream = torch.cuda.current_stream()
    for call, (T, cu, seed) in enumerate([(333, [0, 100, 101, 333], 21),
                                          (200, [0, 64, 200], 22)]):
        # the fixed 256-byte array selects the tensor-core single-kernel plan
        assert gdr.gdr_prefill_plan(len(cu) - 1, T, 3, 128, 128, gate, gdr.GDR_BF16,
                                    256) == gdr.GDR_PATH_TCGEN05
        inp = I.make_inputs(total_T=T, H=3, d_k=128, cu_seqlens=cu, gate_mode=mode,
                            io_dtype=torch.bfloat16, c=0.1, h0_std=0.02, seed=seed)
        d = {k: (None if x is None else x.cuda()) for k, x in dict(
            q=inp.q, k=inp.k, v=inp.v, g=inp.g, beta=inp.beta, h0=inp.h0,
            cu=inp.cu_seqlens).items()}
        o_ref, f_ref = gdr.gdr_prefill_chunked(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"],
                                               d["cu"])
        o = torch.full_like(o_ref, float("nan"))
        fin = torch.full_like(f_ref, float("nan"))
        st = _noalloc_call(d, inp, gate, o, fin, stream)
        assert st == gdr.GDR_OK, gdr.gdr_status_string(st)
        st = lib.gdr_prefill_noalloc_check(ctypes.c_void_p(stream.cuda_stream))
        assert st == gdr.GDR_OK, gdr.gdr_status_string(st)
        # against the fp64 oracle, at the contract tolerances
        o64, f64 = oracle_prefill(inp)
        check(inp, o, fin, o64, f64, f"noalloc {mode} call {call}")
        # and against the workspace entry point on the same inputs
        err_o = float((o.float() - o_ref.float()).abs().max())
        assert err_o <= TOL_BF16_O, (call, err_o)
        f, fr = fin.cpu().numpy(), f_ref.cpu().numpy()
        per = max(rel_frob(f[n, h], fr[n, h]) for n in range(inp.num_seqs) for h in range(inp.H))
        assert per <= TOL_BF16_STATE_REL, (call, per)
        assert not np.isnan(f).any()


def test_noalloc_check_reports_a_wait_that_gave_up_once():
    """A bounded wait on a flag that nothing sets gives up after 1,000 polls
    and records the failure in the fixed array; the check reports it as a
    device timeout, clears it, and the next check reports nothing."""
    lib = gdr.load_library()
    stream = torch.cuda.current_stream()
    sp = ctypes.c_void_p(stream.cuda_stream)
    assert lib.gdr_prefill_noalloc_check(sp) == gdr.GDR_OK
    assert lib.gdr_test_noalloc_wait_timeout(1000, sp) == gdr.GDR_OK
    assert lib.gdr_prefill_noalloc_check(sp) == gdr.GDR_ERR_DEVICE_TIMEOUT
    assert lib.gdr_prefill_noalloc_check(sp) == gdr.GDR_OK
    # the Python binding raises on the same report
    assert lib.gdr_test_noalloc_wait_timeout(1000, sp) == gdr.GDR_OK
    with pytest.raises(gdr.GdrError):
        gdr.gdr_prefill_noalloc_check(stream)
    gdr.gdr_prefill_noalloc_check(stream)
    assert lib.gdr_test_noalloc_wait_timeout(0, sp) == gdr.GDR_ERR_INVALID_ARG


def test_noalloc_rejects_invalid_arguments_like_the_workspace_entry_point():
    lib = gdr.load_library()
    st = lib.gdr_prefill_chunked_noalloc(None, None, None, None, None, None, None, 1, 64, 2, 128,
                                         128, 0, 1, None, None, None)
    assert st == gdr.GDR_ERR_INVALID_ARG
