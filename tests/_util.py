"""Shared helpers for the parity tests: move a workload to the GPU, run the
library through its C ABI, run the oracle, and compare with the tolerances
of the contract:

* fp32 I/O: max |GPU - oracle| <= 1e-4 on o and on the final state;
* bf16 q/k/v: max |GPU - oracle| <= 2e-2 on o, and relative Frobenius error
  <= 1e-3 on the fp32 final state, per (sequence, head) and overall.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from gated_delta_rule_151_b200 import gdr

TOL_F32 = 1e-4
TOL_BF16_O = 2e-2
TOL_BF16_STATE_REL = 1e-3


def to_device(inp, device="cuda"):
    d = {
        "q": inp.q.to(device), "k": inp.k.to(device), "v": inp.v.to(device),
        "g": inp.g.to(device), "beta": inp.beta.to(device),
        "h0": None if inp.h0 is None else inp.h0.to(device),
        "cu": inp.cu_seqlens.to(device),
    }
    return d


# Workspace that selects each tcgen05 plan: None lets the binding allocate the
# reported size (the chunk-parallel plan where it applies); 16 bytes is the
# single-kernel plan's minimum.
PLANS = ("split", "single")


def plan_workspace(plan):
    if plan == "single":
        return torch.zeros(16, dtype=torch.uint8, device="cuda")
    return None


def gpu_prefill(inp, use_cu=True, initial_state="h0", final_state=None, plan="split"):
    d = to_device(inp)
    h0 = d["h0"] if initial_state == "h0" else initial_state
    fn = gdr.gdr_prefill_chunked if inp.H_qk == inp.H else gdr.gdr_prefill_chunked_gqa
    ws = plan_workspace(plan)
    o, fin = fn(d["q"], d["k"], d["v"], d["g"], d["beta"], h0, d["cu"] if use_cu else None,
                num_seqs=inp.num_seqs, final_state=final_state, workspace=ws)
    torch.cuda.synchronize()
    if ws is not None:
        gdr.gdr_prefill_check_workspace(ws)
    return o, fin


def oracle_prefill(inp, heads=None, seqs=None):
    return oracle.loop.run_inputs(inp, heads=heads, seqs=seqs)


def rel_frob(a: np.ndarray, b: np.ndarray) -> float:
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a - b))


def check(inp, o_gpu, fin_gpu, o_ref, fin_ref, label="", state_rel_tol=TOL_BF16_STATE_REL):
    """Assert the contract tolerances (a case may pass a derived state
    tolerance, stating why); returns the error summary."""
    o = o_gpu.float().cpu().numpy().astype(np.float64) if torch.is_tensor(o_gpu) else o_gpu
    f = fin_gpu.float().cpu().numpy().astype(np.float64) if torch.is_tensor(fin_gpu) else fin_gpu
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.all(np.isfinite(o)), f"{label}: non-finite output"
    err_o = float(np.max(np.abs(o - o_ref))) if o.size else 0.0
    out = {"max_abs_o": err_o}
    if fin_ref is not None:
        assert f.shape == fin_ref.shape
        assert np.all(np.isfinite(f)), f"{label}: non-finite state"
        err_s = float(np.max(np.abs(f - fin_ref))) if f.size else 0.0
        out["max_abs_state"] = err_s
        per = [rel_frob(f[n, h], fin_ref[n, h]) for n in range(f.shape[0]) for h in range(f.shape[1])]
        out["rel_frob_state_max"] = max(per) if per else 0.0
        out["rel_frob_state"] = rel_frob(f, fin_ref) if f.size else 0.0
    if inp.io_dtype == torch.float32:
        assert err_o <= TOL_F32, f"{label}: o max-abs {err_o}"
        if fin_ref is not None:
            assert out["max_abs_state"] <= TOL_F32, f"{label}: state max-abs {out['max_abs_state']}"
    else:
        assert err_o <= TOL_BF16_O, f"{label}: o max-abs {err_o}"
        if fin_ref is not None:
            assert out["rel_frob_state_max"] <= state_rel_tol, f"{label}: {out}"
            assert out["rel_frob_state"] <= state_rel_tol, f"{label}: {out}"
    return out
