"""Several decode tokens per sequence in one pass over the state (draft
verification for speculative decoding) against the fp64 oracle, against T
single-token steps (bit for bit: same arithmetic in the same order), and
with per-token state snapshots for rollback."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_151_b200 import gdr
from gated_delta_rule_151_b200 import inputs as I
from _util import TOL_BF16_O, TOL_BF16_STATE_REL, TOL_F32, rel_frob

pytestmark = pytest.mark.gpu


def _inputs(N, T, H, Hqk, d, mode, io, seed):
    inp = I.make_inputs(total_T=N * T, H=H, H_qk=Hqk, d_k=d, num_seqs=N, gate_mode=mode,
                        io_dtype=io, c=0.2, h0_std=0.05, seed=seed)
    dev = "cuda"
    shp = lambda x: x.reshape(N, T, *x.shape[1:]).to(dev)
    return inp, shp(inp.q), shp(inp.k), shp(inp.v), shp(inp.g), shp(inp.beta)


@pytest.mark.parametrize("T", [1, 3, 4, 8])
@pytest.mark.parametrize("mode", [I.SCALAR, I.CHANNEL])
@pytest.mark.parametrize("d,io", [(128, torch.bfloat16), (32, torch.float32)])
def test_decode_multi_matches_oracle_with_snapshots(T, mode, d, io):
    N, H, Hqk = 3, 4, 2
    inp, q, k, v, g, b = _inputs(N, T, H, Hqk, d, mode, io, seed=50 + T)
    state = inp.h0.cuda().clone()
    snaps = torch.full((N, T, H, d, d), float("nan"), device="cuda")
    o = gdr.gdr_decode_multi(q, k, v, g, b, state, snapshots=snaps)
    torch.cuda.synchronize()
    o_ref, f_ref = oracle.loop.run_inputs(inp)                 # sequences of T tokens
    o_ref = o_ref.reshape(N, T, H, d)
    o_np, f_np = o.float().cpu().numpy(), state.cpu().numpy()
    tol_o = TOL_F32 if io == torch.float32 else TOL_BF16_O
    assert np.max(np.abs(o_np - o_ref)) <= tol_o
    if io == torch.float32:
        assert np.max(np.abs(f_np - f_ref)) <= TOL_F32
    else:
        assert max(rel_frob(f_np[n, h], f_ref[n, h]) for n in range(N) for h in range(H)) <= TOL_BF16_STATE_REL
    s_np = snaps.cpu().numpy()
    assert np.array_equal(s_np[:, T - 1], f_np)                # last snapshot = final state
    for t in range(T - 1):                                     # earlier snapshots vs truncated runs
        cu = [0]
        sub = I.make_inputs(total_T=N * T, H=H, H_qk=Hqk, d_k=d, num_seqs=N, gate_mode=mode,
                            io_dtype=io, c=0.2, h0_std=0.05, seed=50 + T)
        sel = np.concatenate([np.arange(n * T, n * T + t + 1) for n in range(N)])
        _, f_t = oracle.run(sub.q[sel], sub.k[sel], sub.v[sel], sub.g[sel], sub.beta[sel], sub.h0,
                            np.arange(N + 1) * (t + 1), channel_gate=(mode == I.CHANNEL))
        if io == torch.float32:
            assert np.max(np.abs(s_np[:, t] - f_t)) <= TOL_F32
        else:
            assert max(rel_frob(s_np[n, t, h], f_t[n, h]) for n in range(N) for h in range(H)) <= TOL_BF16_STATE_REL


@pytest.mark.parametrize("mode", [I.SCALAR, I.CHANNEL])
def test_decode_multi_equals_single_steps(mode):
    N, T, H, Hqk, d = 4, 5, 6, 3, 128
    inp, q, k, v, g, b = _inputs(N, T, H, Hqk, d, mode, torch.bfloat16, seed=60)
    s1 = inp.h0.cuda().clone()
    o1 = gdr.gdr_decode_multi(q, k, v, g, b, s1)
    s2 = inp.h0.cuda().clone()
    o2 = torch.stack([gdr.gdr_decode_step_gqa(q[:, t].contiguous(), k[:, t].contiguous(),
                                              v[:, t].contiguous(), g[:, t].contiguous(),
                                              b[:, t].contiguous(), s2) for t in range(T)], dim=1)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_full_size_draft_verification_sampled():
    """The full 256 x 32 x 128 x 128 (512 MiB) state verified 4 drafts per
    launch, 128 launches, in the launch configuration the benchmark times;
    the oracle checks 16 sequences (all heads) at every token and their final
    states."""
    inp = I.workload("decode_spec_gdn")
    N, T, H, dv = inp.num_seqs, I.SPEC_DRAFT, inp.H, inp.d_v
    L = inp.total_T // N
    steps = L // T
    dev = "cuda"

    def grp(x):   # [N*L, ...] -> [steps, N, T, ...]
        return x.reshape(N, steps, T, *x.shape[1:]).transpose(0, 1).contiguous().to(dev)

    q, k, v, g, b = (grp(x) for x in (inp.q, inp.k, inp.v, inp.g, inp.beta))
    state = inp.h0.to(dev).clone()
    o = torch.empty((steps, N, T, H, dv), dtype=inp.io_dtype, device=dev)
    for s in range(steps):
        gdr.gdr_decode_multi(q[s], k[s], v[s], g[s], b[s], state, o=o[s])
    torch.cuda.synchronize()
    seqs = list(range(0, N, N // 16))
    o_ref, fin_ref = oracle.loop.run_inputs(inp, seqs=seqs)
    o_ref = o_ref.reshape(len(seqs), L, H, dv)
    o_gpu = o.permute(1, 0, 2, 3, 4).reshape(N, L, H, dv)[seqs].float().cpu().numpy()
    err = float(np.max(np.abs(o_gpu - o_ref)))
    assert err <= TOL_BF16_O, err
    fin = state.cpu().numpy()
    per = max(rel_frob(fin[s, h], fin_ref[i, h]) for i, s in enumerate(seqs) for h in range(H))
    assert per <= TOL_BF16_STATE_REL, per
