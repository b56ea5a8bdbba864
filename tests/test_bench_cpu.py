"""Host logic of bench.py on the CPU: the reference arm's JSON line, the
launch accounting of the pipelined chunk-parallel plan, and the algorithmic
byte counts of the workloads (the roofline numerators), each against a count
done by hand here."""
import json
import os
import subprocess
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from gated_delta_rule_151_b200 import inputs as I  # noqa: E402


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "1", "--workloads", "tiny_gdn"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["dtype"] == "f64"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_pipelined_plan_launch_accounting():
    # one launch numbers the chunks; 16 chains of 128 chunks: one prep launch
    # over every chunk, then the segmented scan (6 segments): phase 1, the
    # composition, phase 2
    assert bench.split_launches(I.workload("gdn_prefill")) == 1 + 1 + 3
    # 64 chains of 98,848-byte records, at most 8 GiB per window: 2715 global
    # chunks of 32 heads.  The two equal sequences go without cu_seqlens, so
    # the plan knows each has 512 chunks (1024 in all): one window, in 10
    # pipelined pieces (12, 16, 21, 27, 35, 46, 60, 78, 101 and the last 116)
    kda = I.workload("kda_prefill")
    assert (8 << 30) // (32 * 98848) == 2715
    assert bench.split_launches(kda) == 1 + 2 * 10
    # 48 chains at the gdn_prefill length: three segments (48 x 3 = 144 CTAs
    # in the first phase fit the 148 SMs), the same five launches
    assert bench.split_launches(I.workload("gqa_prefill")) == 1 + 1 + 3
    # 50 chains: three segments no longer fit, pieces of 12, 16, 21, 28, 37
    # and the last 14, each one prep and one chain launch
    wide = I.make_inputs(total_T=8192, H=50, d_k=16, num_seqs=1, gate_mode=I.SCALAR,
                         io_dtype=torch.bfloat16, seed=0)
    assert bench.split_launches(wide) == 1 + 12
    # varlen: 128 chains run by windows; packed lengths bound the chunks by
    # 262144 / 64 + 8 = 4104, within one window of 5431 global chunks of 16
    # heads
    assert (8 << 30) // (16 * 98848) == 5431
    assert bench.split_launches(I.workload("varlen_gdn")) == 1 + 2


def test_prologue_bytes_per_launch():
    case = bench.PrologueCase("prologue_gdn", torch.device("cpu"), seed=0)
    T, C = 8192, 3 * 16 * 128
    expect = (2 * T * C * 2          # x_q, x_k, x_v in; q, k, v out (bf16)
              + C * 4 * 4            # taps
              + 2 * T * 16 * 4       # x_g in, g out
              + 2 * T * 16 * 4       # x_beta in, beta out
              + 16 * 4               # gate coefficients
              + 2 * C * 3 * 4)       # convolution state in and out
    assert case.bytes == expect


def test_backward_bytes_per_launch():
    case = bench.BackwardCase("backward_gdn", torch.device("cpu"), seed=0)
    T, H, d = 8192, 16, 128
    act = T * H * d
    expect = (4 * act * 2            # q, k, v, dO (bf16)
              + 2 * T * H * 4        # g in, dg out
              + 2 * T * H * 4        # beta in, dbeta out
              + H * d * d * 4        # dS_final
              + 3 * act * 4          # dq, dk, dv (fp32)
              + H * d * d * 4)       # d_initial_state
    assert case.bytes == expect
    # the chunked form's records: 475,648 bytes per (chunk, head) for up to
    # T / 64 + 1 chunks (cu_seqlens given), after 256 bytes of chunk offsets
    assert case.ws.numel() == 256 + (T // 64 + 1) * H * 475648
    # the chunked form's products, per (chunk, head): prep 3.67 M, chains
    # 4.19 M, local 7.86 M multiply-adds (d = 128, C = 64), over 128 x 16
    macs = (2 * 64 * 64 * 128 * 2 + 128 * 128 * 64 + 64 * 128 * 64
            + 4 * 128 * 128 * 64
            + 3 * 64 * 128 * 128 + 8 * 64 * 64 * 128 + 2 * 64 ** 3)
    assert macs == 15_728_640
    assert case.flops == 2 * macs * (T // 64) * H
    # no chunked form for the channel gate: no flop count
    kda = I.make_inputs(total_T=128, H=2, d_k=128, num_seqs=1, gate_mode=I.CHANNEL, seed=1)
    assert bench.backward_flops(kda) == 0


def test_reference_arm_under_two_ranks_prints_once():
    # launched like the multi-GPU bench: rank 0 alone times the oracle and
    # prints; the other rank exits 0 without work
    import socket
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                        "--nproc-per-node", "2", "--master-addr", "127.0.0.1", "--master-port",
                        str(port), os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "1", "--workloads", "tiny_gdn"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2
