"""The multi-GPU path on the CPU: two gloo ranks.  Sequences and heads are
independent, so ranks process separate batches with no data-path exchange;
the only collective is the max over ranks of the step time, and the job
throughput is every rank's tokens over that max."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from gated_delta_rule_151_b200 import inputs as I


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    import bench
    # each rank: its own batch (seeded by rank), run through the oracle here
    inp = I.workload("tiny_gdn", seed=rank)
    o, fin = oracle.loop.run_inputs(inp, nthreads=1)
    ms_local = 10.0 + 5.0 * rank          # pretend step times
    value, ms = bench.aggregate_throughput(inp.total_T, ms_local, ws, device="cpu")
    digest = torch.tensor([float(np.abs(o).sum())], dtype=torch.float64)
    gathered = [torch.zeros(1, dtype=torch.float64) for _ in range(ws)]
    dist.all_gather(gathered, digest)
    out[rank] = (value, ms, [float(g.item()) for g in gathered])
    dist.destroy_process_group()


def test_two_ranks_weak_scaling_accounting():
    ws = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(ws, port, out), nprocs=ws, join=True)
        res = dict(out)
    for rank in range(ws):
        value, ms, digests = res[rank]
        assert ms == 15.0                             # the slowest rank's time
        assert abs(value - 2 * 64 / 0.015) < 1e-6     # all ranks' tokens / max time
        assert digests[0] != digests[1]               # ranks really had different batches
