"""Benchmark of the gated delta-rule library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workloads a,b,...]
                    [--impl ours|reference]

Prints ONE JSON line on rank 0.  The headline (`value`) is the first
workload; by default that is the largest single-GPU configuration, the
long-context variable-length GDN prefill (8 packed sequences, 262,144 tokens,
16 heads, d = 128, bf16).  The other benchmark configurations (the 1 x 8192
GDN prefill, the 2 x 32768 KDA prefill with an initial state, the
256-sequence x 512-step GDN and KDA decodes, and the 1 x 8192 GDN prefill
from raw projections with the input-side prologue fused into it) follow
under "workloads", each with the same fields: its own roofline, end-to-end
figure, clock record and (where the recurrence oracle runs it) CPU baseline.

A "step" is one pass of the whole hot path over one batch of synthetic input:
one gdr_prefill_chunked call for a prefill workload, the 512 consecutive
gdr_decode_step calls for a decode workload, one gdr_prologue call for the
prologue workload, one gdr_prefill_fused call for the fused workload.  Timing: W untimed warm-up steps, then one step is
captured as a CUDA graph, and K replays of it are each timed with CUDA events
on the stream the kernels are launched on (--no-graph times eager calls
instead, which adds the host's per-call time whenever it exceeds the GPU's);
an L2 flush (a 512 MiB write, then a read of it, so that the flush's own
dirty lines are written back before the timed region) precedes every timed
step and is not timed.
The end-to-end figure (`e2e`) always goes through the Python binding with
pinned host buffers, host/device copies inside its timed region.  Barrier + synchronize bracket the timed region; the time is the
max over ranks.  For N > 1 every rank runs its own independent batch (heads
and sequences are independent; no collective on the data path) and `value`
is the sum of tokens over ranks divided by that time ("weak" scaling).

--impl reference times the fp64 CPU oracle (the reference this library is
checked against) on a bounded sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_delta_rule_151_b200 import gdr  # noqa: E402
from gated_delta_rule_151_b200 import inputs as I  # noqa: E402

METRIC = "gated delta-rule tokens/s (prefill, decode) and % roofline at 1 B200"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CHUNK = 64
# the five benchmark configurations that run on the GPU (the tiny GDN case is
# a parity-only configuration); the first is the headline
DEFAULT_WORKLOADS = "varlen_gdn,gdn_prefill,kda_prefill,decode_gdn,decode_kda,prefill_fused_gdn,backward_gdn"


# ------------------------------------------------------------ plumbing ----

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class NvmlClockSampler:
    """SM clock and clock-event reasons read through NVML every 20 ms while
    running (read-only queries; no setting is changed).  Short timed regions
    still get several samples."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))

    def __init__(self, gpu_index: int, period_s: float = 0.02):
        import pynvml
        self.nv = pynvml
        self.gpu = gpu_index
        self.period = period_s
        self.samples = []
        self._stop = threading.Event()

    def __enter__(self):
        nv = self.nv
        nv.nvmlInit()
        uuid = torch.cuda.get_device_properties(self.gpu).uuid
        self.h = None
        try:
            self.h = nv.nvmlDeviceGetHandleByUUID("GPU-" + str(uuid))
        except Exception:
            self.h = nv.nvmlDeviceGetHandleByIndex(self.gpu)
        self.smax = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()
        return self

    def _sample(self):
        nv = self.nv
        sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except AttributeError:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.samples.append((sm, r))

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        self.t.join(timeout=2)
        self._sample()
        try:
            self.nv.nvmlShutdown()
        except Exception:
            pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = sorted({n for _, r in self.samples for n, bit in self.REASONS if r & bit})
        return {"sm_mhz": statistics.median(s for s, _ in self.samples),
                "sm_max_mhz": self.smax, "reasons": reasons, "samples": len(self.samples),
                "source": "NVML every 20 ms during the timed region"}


def clock_sampler(gpu_index: int):
    """NVML sampler where NVML is importable, else nvidia-smi at 200 ms."""
    try:
        import pynvml  # noqa: F401
        return NvmlClockSampler(gpu_index)
    except Exception:
        return ClockSampler(gpu_index)


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            t_end = time.time() + 5.0            # let the sampler come up first
            while not self.lines and time.time() < t_end and self.proc.poll() is None:
                time.sleep(0.05)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.t.join(timeout=2)

    def summary(self):
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


def l2_flusher(device):
    """Write 512 MiB (four times the 126 MB L2), then read it back: the write
    evicts every line the last step left, and the read pass makes the write's
    own dirty lines go back to HBM here, outside the timed region, instead of
    inside the next timed step."""
    buf = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=device)
    sink = torch.empty((), dtype=torch.int64, device=device)

    def flush():
        buf.fill_(1)
        torch.amax(buf.view(torch.int64), dim=0, out=sink)
    return flush


# ------------------------------------------------------- work per step ----

def io_bytes(dtype):
    return 2 if dtype == torch.bfloat16 else 4


def prefill_work(inp):
    """Algorithmic bytes and flops of one prefill launch (per-token-head
    figures: q, k, v read, o written, beta and g read; plus 64 KiB of fp32
    state written per (sequence, head), and read when an initial state is
    given)."""
    T, H, dk, dv, N = inp.total_T, inp.H, inp.d_k, inp.d_v, inp.num_seqs
    e = io_bytes(inp.io_dtype)
    gate = 4 * (dk if inp.gate_mode == I.CHANNEL else 1)
    # q and k per query/key head; v, o, beta, g per value head
    per_t = inp.H_qk * e * 2 * dk + H * (e * 2 * dv + 4 + gate)
    state = 4 * dk * dv * N * H * (2 if inp.h0 is not None else 1)
    byts = T * per_t + state
    flops = T * H * (5 * CHUNK * max(dk, dv) + 6 * dk * dv)
    return byts, flops


def decode_work(inp):
    """Algorithmic bytes of one decode launch (one token per sequence): the
    fp32 state read and written once, q/k/v/beta/g read, o written."""
    N, H, dk, dv = inp.num_seqs, inp.H, inp.d_k, inp.d_v
    e = io_bytes(inp.io_dtype)
    gate = 4 * (dk if inp.gate_mode == I.CHANNEL else 1)
    return N * H * (2 * 4 * dk * dv + e * (2 * dk + 2 * dv) + 4 + gate)


def split_launches(inp):
    """Kernel launches of the chunk-parallel plan, mirroring its plan: one
    launch that numbers every sequence's chunks, then a prep and a chain kernel
    per window of chunks (a window holds at most 8 GiB of records at 98,848
    bytes per chunk and head), or, when one window holds every record and
    there are at most 64 (sequence, head) chains, per pipeline piece, or, with
    at most 49 chains, one prep launch and the three launches of the
    segmented scan."""
    chains = inp.num_seqs * inp.H
    # equal lengths go without cu_seqlens, so the library knows each
    # sequence's length; otherwise total_T bounds it
    equal = inp.equal_lengths()
    longest = inp.total_T // inp.num_seqs if equal else inp.total_T
    max_chunks = -(-longest // 64)
    max_total = inp.num_seqs * max_chunks if equal else -(-inp.total_T // 64) + inp.num_seqs
    window = min(max_total, (8 << 30) // (inp.H * 98848))
    windows = -(-max_total // window)
    if windows > 1 or chains > 64:
        return 1 + 2 * windows
    nseg = min(8, (148 // chains + 3) // 2)
    if nseg >= 3 and max_chunks >= 2 * nseg:
        # few chains: the prep kernel over every chunk, then the segmented scan
        # (segments from zero and their transitions, composition, segments in
        # full from their incoming states)
        return 1 + 1 + 3
    pieces, c, size = 0, 0, 12   # pieces of 12, 16, 21, 27, ... chunks (1.3x growth)
    while c < max_chunks and pieces < 32:
        c = max_chunks if pieces + 1 == 32 else min(c + size, max_chunks)
        pieces += 1
        size = (size * 13 + 9) // 10
    return 1 + 2 * pieces


class PrefillCase:
    kind = "prefill"

    def __init__(self, name, device, seed):
        self.name = name
        self.inp = inp = I.workload(name, seed=seed)
        self.dev = device
        # equal-length batches go in the dense layout (no cu_seqlens), as a
        # caller with a [B, T, H, d] batch would pass them
        self.equal = inp.equal_lengths()
        self.d = {k: (None if v is None else v.to(device)) for k, v in dict(
            q=inp.q, k=inp.k, v=inp.v, g=inp.g, beta=inp.beta, h0=inp.h0,
            cu=None if self.equal else inp.cu_seqlens).items()}
        self.o = torch.empty((inp.total_T, inp.H, inp.d_v), dtype=inp.io_dtype, device=device)
        self.fin = torch.empty((inp.num_seqs, inp.H, inp.d_v, inp.d_k), dtype=torch.float32,
                               device=device)
        gate = gdr.GDR_GATE_CHANNEL if inp.gate_mode == I.CHANNEL else gdr.GDR_GATE_SCALAR
        io = gdr.GDR_BF16 if inp.io_dtype == torch.bfloat16 else gdr.GDR_F32
        nbytes = gdr.gdr_prefill_workspace_size(inp.num_seqs, inp.total_T, inp.H, inp.d_k,
                                                inp.d_v, gate, io)
        self.ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device) if nbytes else None
        self.path = gdr.gdr_prefill_plan(inp.num_seqs, inp.total_T, inp.H, inp.d_k, inp.d_v,
                                         gate, io, nbytes)
        self.bytes, self.flops = prefill_work(inp)
        self.tokens = inp.total_T
        self.launches = split_launches(inp) if self.path == gdr.GDR_PATH_TCGEN05_SPLIT else 1

    def _fn(self):
        return gdr.gdr_prefill_chunked if self.inp.H_qk == self.inp.H else gdr.gdr_prefill_chunked_gqa

    def step(self, stream=None):
        d = self.d
        self._fn()(d["q"], d["k"], d["v"], d["g"], d["beta"], d["h0"], d["cu"],
                   num_seqs=self.inp.num_seqs, o=self.o, final_state=self.fin,
                   workspace=self.ws, stream=stream)

    def host_inputs(self):
        inp = self.inp
        xs = dict(q=inp.q, k=inp.k, v=inp.v, g=inp.g, beta=inp.beta)
        if not self.equal:
            xs["cu"] = inp.cu_seqlens
        if inp.h0 is not None:
            xs["h0"] = inp.h0
        return {k: v.pin_memory() for k, v in xs.items()}

    def e2e_step(self, host, host_o, host_fin, stream):
        dev = {k: v.to(self.dev, non_blocking=True) for k, v in host.items()}
        self._fn()(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev.get("h0"), dev.get("cu"),
                   num_seqs=self.inp.num_seqs, o=self.o, final_state=self.fin,
                   workspace=self.ws, stream=stream)
        host_o.copy_(self.o, non_blocking=True)
        host_fin.copy_(self.fin, non_blocking=True)

    def e2e_buffers(self):
        host = self.host_inputs()
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        ho = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        hf = torch.empty(self.fin.shape, dtype=self.fin.dtype).pin_memory()
        d2h = ho.numel() * ho.element_size() + hf.numel() * hf.element_size()
        return host, ho, hf, h2d, d2h

    def dtype_label(self):
        if self.path in (gdr.GDR_PATH_TCGEN05, gdr.GDR_PATH_TCGEN05_SPLIT):
            return "bf16/tf32 tensor-core operands, fp32 accumulate and state"
        return "f32"


class DecodeCase:
    kind = "decode"

    def __init__(self, name, device, seed):
        self.name = name
        self.inp = inp = I.workload(name, seed=seed)
        self.dev = device
        N = inp.num_seqs
        self.steps = inp.total_T // N
        self.q, self.k, self.v = (I.decode_view(x, N).to(device) for x in (inp.q, inp.k, inp.v))
        self.g = I.decode_view(inp.g, N).to(device)
        self.beta = I.decode_view(inp.beta, N).to(device)
        self.state = inp.h0.to(device).clone()
        self.o = torch.empty((self.steps, N, inp.H, inp.d_v), dtype=inp.io_dtype, device=device)
        self.bytes = decode_work(inp)          # per launch
        self.flops = 0
        self.tokens = inp.total_T              # N * steps per bench step
        self.launches = self.steps
        self.path = None

    def step(self, stream=None):
        for t in range(self.steps):
            gdr.gdr_decode_step(self.q[t], self.k[t], self.v[t], self.g[t], self.beta[t],
                                self.state, o=self.o[t], stream=stream)

    def e2e_buffers(self):
        host = {k: v.cpu().pin_memory() for k, v in
                dict(q=self.q, k=self.k, v=self.v, g=self.g, beta=self.beta).items()}
        ho = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = ho.numel() * ho.element_size()
        self._dev_tok = {k: torch.empty(v.shape[1:], dtype=v.dtype, device=self.dev)
                         for k, v in host.items()}
        return host, ho, None, h2d, d2h

    def e2e_step(self, host, host_o, host_fin, stream):
        dt = self._dev_tok
        for t in range(self.steps):
            for key in dt:
                dt[key].copy_(host[key][t], non_blocking=True)
            gdr.gdr_decode_step(dt["q"], dt["k"], dt["v"], dt["g"], dt["beta"], self.state,
                                o=self.o[t], stream=stream)
            host_o[t].copy_(self.o[t], non_blocking=True)

    def dtype_label(self):
        return "f32"


class SpecDecodeCase(DecodeCase):
    """Draft verification: each launch applies SPEC_DRAFT consecutive tokens of
    every sequence (gdr_decode_multi); a step is the 512 tokens of each
    sequence, i.e. 512 / SPEC_DRAFT launches."""

    def __init__(self, name, device, seed):
        self.name = name
        self.inp = inp = I.workload(name, seed=seed)
        self.dev = device
        N, T = inp.num_seqs, I.SPEC_DRAFT
        L = inp.total_T // N
        self.T, self.steps = T, L // T

        def grp(x):   # [N*L, ...] -> [steps, N, T, ...] contiguous per launch
            return x.reshape(N, self.steps, T, *x.shape[1:]).transpose(0, 1).contiguous().to(device)
        self.q, self.k, self.v, self.g, self.beta = (grp(x) for x in (inp.q, inp.k, inp.v, inp.g,
                                                                      inp.beta))
        self.state = inp.h0.to(device).clone()
        self.o = torch.empty((self.steps, N, T, inp.H, inp.d_v), dtype=inp.io_dtype, device=device)
        e = io_bytes(inp.io_dtype)
        gate = 4 * (inp.d_k if inp.gate_mode == I.CHANNEL else 1)
        self.bytes = N * inp.H * (2 * 4 * inp.d_k * inp.d_v +
                                  T * (e * (2 * inp.d_k + 2 * inp.d_v) + 4 + gate))
        self.flops = 0
        self.tokens = inp.total_T
        self.launches = self.steps
        self.path = None

    def step(self, stream=None):
        for t in range(self.steps):
            gdr.gdr_decode_multi(self.q[t], self.k[t], self.v[t], self.g[t], self.beta[t],
                                 self.state, o=self.o[t], stream=stream)

    def e2e_buffers(self):
        host = {k: v.cpu().pin_memory() for k, v in
                dict(q=self.q, k=self.k, v=self.v, g=self.g, beta=self.beta).items()}
        ho = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = ho.numel() * ho.element_size()
        self._dev_tok = {k: torch.empty(v.shape[1:], dtype=v.dtype, device=self.dev)
                         for k, v in host.items()}
        return host, ho, None, h2d, d2h

    def e2e_step(self, host, host_o, host_fin, stream):
        dt = self._dev_tok
        for t in range(self.steps):
            for key in dt:
                dt[key].copy_(host[key][t], non_blocking=True)
            gdr.gdr_decode_multi(dt["q"], dt["k"], dt["v"], dt["g"], dt["beta"], self.state,
                                 o=self.o[t], stream=stream)
            host_o[t].copy_(self.o[t], non_blocking=True)


class PrologueCase:
    """The input-side prologue at the gdn_prefill shape: one gdr_prologue
    launch per step (convolution with state, SiLU, q/k normalisation, gate
    and beta maps)."""
    kind = "prologue"
    kernel_label = "prologue"

    def __init__(self, name, device, seed):
        self.name = name
        self.inp = inp = I.prologue_workload(name, seed=seed)
        self.dev = device
        self.d = {k: getattr(inp, k).to(device) for k in
                  ("xq", "xk", "xv", "wq", "wk", "wv", "xg", "gscale", "xb", "conv_state")}
        N = inp.num_seqs
        self.Call = inp.wq.shape[0] * 2 + inp.wv.shape[0]
        self.state_out = torch.empty((N, self.Call, 3), dtype=torch.float32, device=device)
        e = io_bytes(inp.io_dtype)
        T, Call = inp.total_T, self.Call
        gate = inp.xg.numel() * 4
        # read x (q, k, v), taps, gate and beta inputs, state; write the same shapes back
        self.bytes = (2 * T * Call * e + Call * 16 + 2 * gate + 2 * T * inp.H * 4 + inp.H * 4
                      + 2 * N * Call * 12)
        self.flops = 0
        self.tokens = T
        self.launches = 1
        self.path = None
        self.out = None

    def _call(self, d, stream):
        self.out = gdr.gdr_prologue(d["xq"], d["xk"], d["xv"], d["wq"], d["wk"], d["wv"], d["xg"],
                                    d["gscale"], d["xb"], d["conv_state"], None,
                                    num_seqs=self.inp.num_seqs, conv_state_out=self.state_out,
                                    silu=True, normalize_qk=True,
                                    **({} if self.out is None else dict(
                                        q=self.out[0], k=self.out[1], v=self.out[2],
                                        g=self.out[3], beta=self.out[4])),
                                    stream=stream)

    def step(self, stream=None):
        self._call(self.d, stream)

    def e2e_buffers(self):
        host = {k: v.cpu().pin_memory() for k, v in self.d.items()}
        if self.out is None:
            self.step()
        outs = list(self.out) + [self.state_out]
        ho = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = sum(o.numel() * o.element_size() for o in ho)
        return host, ho, None, h2d, d2h

    def e2e_step(self, host, host_o, host_fin, stream):
        dev = {k: v.to(self.dev, non_blocking=True) for k, v in host.items()}
        self._call(dev, stream)
        for h, o in zip(host_o, list(self.out) + [self.state_out]):
            h.copy_(o, non_blocking=True)

    def dtype_label(self):
        return "f32 arithmetic, bf16 in and out"


class FusedPrefillCase:
    """The prologue fused into the chunked prefill at the gdn_prefill shape:
    one gdr_prefill_fused call per step from the raw projections (the
    prologue_gdn inputs: convolution with state, SiLU, q/k norms, gate and
    beta maps) to o, the final state and the outgoing convolution state."""
    kind = "prefill"
    kernel_label = "tcgen05 chunk-parallel prefill with the prologue fused into its stage step"

    def __init__(self, name, device, seed):
        self.name = name
        self.inp = inp = I.prologue_workload(name, seed=seed)
        self.dev = device
        self.d = {k: getattr(inp, k).to(device) for k in
                  ("xq", "xk", "xv", "wq", "wk", "wv", "xg", "gscale", "xb", "conv_state")}
        N, T, H = inp.num_seqs, inp.total_T, inp.xv.shape[1]
        self.N, self.T, self.H = N, T, H
        self.Call = inp.wq.shape[0] * 2 + inp.wv.shape[0]
        self.state_out = torch.empty((N, self.Call, 3), dtype=torch.float32, device=device)
        self.o = torch.empty((T, H, 128), dtype=torch.bfloat16, device=device)
        self.fin = torch.empty((N, H, 128, 128), dtype=torch.float32, device=device)
        nb = gdr.gdr_prefill_workspace_size(N, T, H, 128, 128, gdr.GDR_GATE_SCALAR, gdr.GDR_BF16)
        self.ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=device)
        e = io_bytes(inp.io_dtype)
        # read the raw projections, taps, raw gate and beta, coefficients and
        # the incoming convolution state; write o, the final state and the
        # outgoing convolution state
        self.bytes = (T * self.Call * e + self.Call * 16 + inp.xg.numel() * 4 + T * H * 4
                      + H * 4 + 2 * N * self.Call * 12 + T * H * 128 * e + N * H * 128 * 128 * 4)
        self.flops = T * H * (5 * CHUNK * 128 + 6 * 128 * 128)
        self.tokens = T
        self.launches = 6
        self.path = None

    def _call(self, d, stream):
        gdr.gdr_prefill_fused(d["xq"], d["xk"], d["xv"], d["wq"], d["wk"], d["wv"], d["xg"],
                              d["gscale"], d["xb"], d["conv_state"], None, None,
                              num_seqs=self.N, conv_state_out=self.state_out, silu=True,
                              normalize_qk=True, o=self.o, final_state=self.fin,
                              workspace=self.ws, stream=stream)

    def step(self, stream=None):
        self._call(self.d, stream)

    def e2e_buffers(self):
        host = {k: v.cpu().pin_memory() for k, v in self.d.items()}
        outs = [self.o, self.fin, self.state_out]
        ho = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = sum(o.numel() * o.element_size() for o in ho)
        return host, ho, None, h2d, d2h

    def e2e_step(self, host, host_o, host_fin, stream):
        dev = {k: v.to(self.dev, non_blocking=True) for k, v in host.items()}
        self._call(dev, stream)
        for h, o in zip(host_o, [self.o, self.fin, self.state_out]):
            h.copy_(o, non_blocking=True)

    def dtype_label(self):
        return "bf16/fp16 tensor-core operands, fp32 accumulate, state and prologue arithmetic"


def backward_flops(inp, C=64):
    """Flops of the chunked gradient's products per step (2 per multiply-add;
    the forms the kernels run, each product once whatever its number of
    split passes).  Per (chunk, head), with d = d_k = d_v:
      prep    K K^T, Q K^T (C C d each), W, U~ (C d C each), Y (d d C), Z (C d C)
      chains  forward W S^T, U^T K^ and reverse K^ L'^T, dU^T W (d d C each)
      local   U L', dU S, dO S (C d d each); dP, T^T dU, T^T dW, the two terms
              of dT, (M + M^T) K, (dP o R) K, (dP o R)^T Q (C C d each);
              dT T^T, T^T Y (C C C each)
    Zero where the chunked form does not apply (it runs the token form)."""
    if inp.gate_mode != I.SCALAR or inp.d_k != 128 or inp.d_v != 128:
        return 0
    d = inp.d_k
    macs = (2 * C * C * d + 2 * C * d * C + d * d * C + C * d * C      # prep
            + 4 * d * d * C                                            # chains
            + 3 * C * d * d + 8 * C * C * d + 2 * C * C * C)           # local
    cu = inp.cu_seqlens.numpy()
    chunks = int(sum((int(cu[n + 1]) - int(cu[n]) + C - 1) // C for n in range(len(cu) - 1)))
    return 2 * macs * chunks * inp.H


class BackwardCase:
    """The gradient of the recurrence at the gdn_prefill shape: one
    gdr_backward call per step (upstream gradients dO and dS_final drawn by
    the input module)."""
    kind = "backward"
    kernel_label = ("backward in chunked form: chunk prep, forward and reverse state chains, "
                    "chunk-local gradients")

    def __init__(self, name, device, seed):
        self.name = name
        self.inp = inp = I.workload("gdn_prefill", seed=seed)
        dO, dsf = I.make_grad_inputs(inp, seed=seed)
        self.dev = device
        self.d = {k: (None if v is None else v.to(device)) for k, v in dict(
            q=inp.q, k=inp.k, v=inp.v, g=inp.g, beta=inp.beta, h0=inp.h0, cu=inp.cu_seqlens,
            dO=dO, dsf=dsf).items()}
        nbytes = gdr.gdr_backward_workspace_size(inp.num_seqs, inp.total_T, inp.H, inp.d_k,
                                                 inp.d_v)
        self.ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
        e = io_bytes(inp.io_dtype)
        T, H, Hqk, dk, dv, N = inp.total_T, inp.H, inp.H_qk, inp.d_k, inp.d_v, inp.num_seqs
        gate = inp.g.numel() * 4
        state = N * H * dv * dk * 4
        # read q, k, v, dO, g, beta, dS_final (h0 when given); write dq, dk, dv (fp32), dg,
        # dbeta, d_initial_state
        self.bytes = (T * (2 * Hqk * dk + 2 * H * dv) * e + 2 * gate + 2 * T * H * 4
                      + (2 if inp.h0 is not None else 1) * state
                      + T * (2 * Hqk * dk + H * dv) * 4 + state)
        self.flops = backward_flops(inp)
        self.tokens = T
        self.launches = 4   # chunk numbering, prep, the two chains in one launch, local gradients
        self.path = None
        self.out = None

    def _call(self, d, stream):
        self.out = gdr.gdr_backward(d["q"], d["k"], d["v"], d["g"], d["beta"], d.get("h0"),
                                    d["cu"], d_o=d["dO"], d_final_state=d.get("dsf"),
                                    workspace=self.ws, stream=stream)

    def step(self, stream=None):
        self._call(self.d, stream)

    def e2e_buffers(self):
        host = {k: v.cpu().pin_memory() for k, v in self.d.items() if v is not None}
        if self.out is None:
            self.step()
        ho = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in self.out if o is not None]
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = sum(o.numel() * o.element_size() for o in ho)
        return host, ho, None, h2d, d2h

    def e2e_step(self, host, host_o, host_fin, stream):
        dev = {k: v.to(self.dev, non_blocking=True) for k, v in host.items()}
        self._call(dev, stream)
        for h, o in zip(host_o, [o for o in self.out if o is not None]):
            h.copy_(o, non_blocking=True)

    def dtype_label(self):
        return "f32 arithmetic and gradients, bf16 inputs"


def make_case(name, device, seed):
    if name == "backward_gdn":
        return BackwardCase(name, device, seed)
    if name == "prologue_gdn":
        return PrologueCase(name, device, seed)
    if name == "prefill_fused_gdn":
        return FusedPrefillCase(name, device, seed)
    if name == "decode_spec_gdn":
        return SpecDecodeCase(name, device, seed)
    if name.startswith("decode"):
        return DecodeCase(name, device, seed)
    return PrefillCase(name, device, seed)


# ----------------------------------------------------------- measuring ----

def timed_steps(fn, K, flush, stream):
    """K steps, each bracketed by CUDA events on `stream` after an untimed
    L2 flush; returns the per-step times in ms."""
    times = []
    for _ in range(K):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        times.append((a, b))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in times]


def max_over_ranks(x, ws, device="cuda"):
    """Max of a per-rank scalar over all ranks (timing only; no data-path
    collective exists)."""
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(tokens_per_rank, ms_local, ws, device="cuda"):
    """Weak scaling: every rank processes its own batch of `tokens_per_rank`
    tokens; the job's throughput is all ranks' tokens over the slowest rank's
    time.  Returns (tokens/s, max ms)."""
    ms = max_over_ranks(ms_local, ws, device)
    return tokens_per_rank * ws / (ms / 1e3), ms


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


def load_traffic(case):
    """DRAM bytes per launch (single-kernel plans) or per step (the two-kernel
    chunk-parallel plan) from a committed ncu capture, if it was taken on the
    kernel sources as they are now."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        ent = d.get(case.name)
        if not ent:
            return None
        import hashlib
        h = hashlib.sha256()
        for rel in ent["sources"]:
            h.update(open(os.path.join(ROOT, rel), "rb").read())
        if h.hexdigest() != ent["sources_sha256"]:
            return None
        # one kernel: DRAM bytes per launch; a multi-kernel plan: per step
        return float(ent.get("bytes_per_step", ent.get("bytes_per_launch")))
    except Exception:
        return None


def capture_step(case, stream):
    """One step captured as a CUDA graph (after warm-up, so every kernel
    attribute and helper stream already exists): replaying it runs exactly the
    step's kernels, back to back, without the host's per-call Python and
    argument-checking time between them."""
    try:
        g = torch.cuda.CUDAGraph(keep_graph=True)   # keep the graph so its nodes can be counted
    except TypeError:
        g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        case.step(stream)
    torch.cuda.synchronize()
    return g


def graph_kernel_nodes(graph):
    """Kernel nodes in a captured step (every kernel launch of the step is one
    node), or None where the graph cannot be inspected."""
    try:
        from cuda.bindings import runtime as rt
        g = rt.cudaGraph_t(init_value=int(graph.raw_cuda_graph()))
        err, _, n = rt.cudaGraphGetNodes(g, 0)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        err, nodes, n = rt.cudaGraphGetNodes(g, n)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        kern = 0
        for node in nodes[:n]:
            err, kind = rt.cudaGraphNodeGetType(node)
            if err == rt.cudaError_t.cudaSuccess and kind == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                kern += 1
        return kern
    except Exception:
        return None


def bench_case(case, args, ws, rank, flush, stream, pk, pk_kind):
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            case.step(stream)
        torch.cuda.synchronize()
        graph = None if args.no_graph else capture_step(case, stream)
        counted = graph_kernel_nodes(graph) if graph is not None else None
        if counted:
            case.launches = counted
        run = graph.replay if graph is not None else (lambda: case.step(stream))
        run()
        torch.cuda.synchronize()
        barrier(ws)
        with clock_sampler(torch.cuda.current_device()) as clk:
            times = timed_steps(run, args.steps, flush, stream)
        barrier(ws)
        del graph
    value, ms = aggregate_throughput(case.tokens, sum(times) / len(times), ws)
    tokens_all = case.tokens * ws
    # decode and the prologue: bytes per launch over the time per launch;
    # prefill and the chunked gradient: the whole step's bytes (every kernel of
    # the plan) over the step time
    launch_ms = ms if case.kind in ("prefill", "backward") else ms / case.launches
    achieved = case.bytes / (launch_ms / 1e3) / 1e9
    hbm_peak = float(pk["hbm_gbs"])
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
            "frac": round(achieved / hbm_peak, 4), "traffic": load_traffic(case),
            "peak_source": f"{pk_kind} HBM copy bandwidth"}
    if case.kind == "prefill":
        tc_peak = float(pk["bf16_tflops"]) / 2.0   # tf32 = half the bf16 rate
        roof["flops_per_launch"] = case.flops
        roof["tensor_tflops"] = round(case.flops / (launch_ms / 1e3) / 1e12, 2)
        roof["tensor_frac_of_tf32_peak"] = round(case.flops / (launch_ms / 1e3) / 1e12 / tc_peak, 4)
        roof["algorithmic_bytes_per_launch"] = case.bytes
    else:
        roof["algorithmic_bytes_per_launch"] = case.bytes
        roof["frac_of_8TBps_nominal"] = round(achieved / 8000.0, 4)
    if case.kind == "backward" and case.flops:
        # the gradient's products are fp32-accurate (split operands on the
        # tensor cores): their useful rate against the CUDA cores' fp32 FMA
        # rate, 148 SMs x 128 lanes x 2 flops at the maximum SM clock
        fma_peak = 148 * 128 * 2 * 1965e6 / 1e12
        rate = case.flops / (launch_ms / 1e3) / 1e12
        roof["flops_per_launch"] = case.flops
        roof["fp32_equivalent_tflops"] = round(rate, 2)
        roof["frac_of_fp32_fma_peak"] = round(rate / fma_peak, 4)
        roof["fp32_fma_peak_tflops"] = round(fma_peak, 1)

    # end to end: pinned host buffers, copies inside the timed region
    host, ho, hf, h2d, d2h = case.e2e_buffers()
    with torch.cuda.stream(stream):
        case.e2e_step(host, ho, hf, stream)
        torch.cuda.synchronize()
        barrier(ws)
        e2e_times = timed_steps(lambda: case.e2e_step(host, ho, hf, stream), args.steps, flush,
                                stream)
        barrier(ws)
    e2e_ms = max_over_ranks(sum(e2e_times) / len(e2e_times), ws)
    inp = case.inp
    cfg = {"workload": case.name, "num_seqs": inp.num_seqs, "total_T": inp.total_T,
           "H": inp.H, "H_qk": inp.H_qk, "d_k": inp.d_k, "d_v": inp.d_v, "gate": inp.gate_mode,
           "io": str(inp.io_dtype).replace("torch.", ""),
           "h0": inp.h0 is not None, "l2": "flushed (512 MiB write, then read back) before every timed step",
           "kernel": getattr(case, "kernel_label", None) or (
               "decode" if case.kind == "decode" else
               {gdr.GDR_PATH_TCGEN05: "tcgen05",
                gdr.GDR_PATH_TCGEN05_SPLIT: "tcgen05 chunk-parallel (prep + chain)"}.get(
                   case.path, "simt"))}
    cfg["launch"] = ("the step's kernels replayed from a CUDA graph captured after warm-up"
                     if not args.no_graph else "eager calls through the Python binding")
    if case.kind == "prefill":
        cfg["launches_per_step"] = case.launches
    cfg["launch_count_source"] = ("kernel nodes of the captured step" if counted
                                  else "the library's launch plan")
    if case.kind == "decode":
        cfg["launches_per_bench_step"] = case.steps
        cfg["tokens_per_sequence_per_launch"] = getattr(case, "T", 1)
    return {
        "value": value, "ms_per_step": ms, "tokens_per_step": tokens_all,
        "dtype": case.dtype_label(), "config": cfg, "roofline": roof,
        "e2e": {"value": tokens_all / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": case.launches * args.steps, "clocks": clk.summary(),
    }


def cpu_baseline_backward(name, budget_s=8.0):
    """The fp64 backward oracle (numpy, one thread), as it stands, on whole
    heads of the gradient workload (all tokens) until about budget_s has
    run; tokens/s scaled to the full workload's head count."""
    from oracle import backward as B
    from threadpoolctl import threadpool_limits
    inp = I.workload("gdn_prefill", seed=0)
    dO, dsf = I.make_grad_inputs(inp, seed=0)
    cu = inp.cu_seqlens.numpy()
    done, dt = 0, 0.0
    with threadpool_limits(limits=1):
        while done < inp.H and dt < budget_s:
            h = slice(done, done + 1)
            t = time.perf_counter()
            B.backward(inp.q[:, h], inp.k[:, h], inp.v[:, h], inp.g[:, h], inp.beta[:, h],
                       None if inp.h0 is None else inp.h0[:, h], cu, dO[:, h],
                       None if dsf is None else dsf[:, h])
            dt += time.perf_counter() - t
            done += 1
    value = inp.total_T * (done / inp.H) / dt
    return {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{name}: {done} of {inp.H} heads, all {inp.total_T} tokens, fp64 numpy "
                      f"backward oracle on one thread, {dt:.2f} s"}


def cpu_baseline(name, budget_s=10.0):
    """The oracle, as it stands, on a bounded sample of the workload: whole
    heads (all tokens of every sequence) until the estimated cost reaches the
    budget.  Returns tokens/s scaled to the full workload's head count (a
    decode workload's tokens are its sequences' tokens: the oracle runs the
    same recurrence token by token)."""
    if name == "backward_gdn":
        return cpu_baseline_backward(name)
    import oracle
    inp = I.workload(name)
    cores = oracle.loop.default_threads()
    per_head_flop = 7.0 * inp.d_k * inp.d_v * inp.total_T
    est_rate = 1.2e9 * cores                      # fp64 flop/s, rough
    nh = int(max(1, min(inp.H, budget_s * est_rate / per_head_flop)))
    heads = list(range(nh))
    t = time.perf_counter()
    oracle.loop.run_inputs(inp, heads=heads, nthreads=cores)
    dt = time.perf_counter() - t
    value = inp.total_T * (nh / inp.H) / dt
    return {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{name}: {nh} of {inp.H} heads, all {inp.total_T} tokens of all "
                      f"{inp.num_seqs} sequences, fp64 C loop, {dt:.2f} s"}


# workloads with a timed oracle: the fp64 C recurrence, or the fp64 backward
# oracle for the gradient (the prologue's oracle is not timed here)
CPU_BASELINE_WORKLOADS = ("tiny_gdn", "gdn_prefill", "kda_prefill", "varlen_gdn", "gqa_prefill",
                          "decode_gdn", "decode_kda", "decode_spec_gdn", "backward_gdn")


def run_reference(args, ws, rank):
    """--impl reference: the fp64 oracle timed on the host cores."""
    if rank != 0:
        return
    import oracle
    name = args.workloads.split(",")[0]
    inp = I.workload(name)
    cores = oracle.loop.default_threads()
    per_head_flop = 7.0 * inp.d_k * inp.d_v * inp.total_T
    nh = int(max(1, min(inp.H, 3.0 * 1.2e9 * cores / per_head_flop)))
    heads = list(range(nh))
    for _ in range(args.warmup if args.warmup < 2 else 1):
        oracle.loop.run_inputs(inp, heads=heads[:1], nthreads=cores)
    times = []
    for _ in range(args.steps):
        t = time.perf_counter()
        oracle.loop.run_inputs(inp, heads=heads, nthreads=cores)
        times.append(time.perf_counter() - t)
    dt = sum(times) / len(times)
    value = inp.total_T * (nh / inp.H) / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": name, "sample_heads": nh, "H": inp.H, "total_T": inp.total_T},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{name}: {nh} of {inp.H} heads per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workloads", default=DEFAULT_WORKLOADS,
                    help="comma list from: " + ",".join(I.WORKLOADS) + " (or 'all')")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time eager calls instead of a CUDA-graph replay of the step")
    args = ap.parse_args()
    if args.workloads == "all":
        args.workloads = ("gdn_prefill,kda_prefill,varlen_gdn,gqa_prefill,decode_gdn,decode_kda,"
                          "decode_spec_gdn,prologue_gdn,backward_gdn")
    if args.warmup < 3:
        args.warmup = 3
    ws, rank, local = dist_env()

    if args.impl == "reference":
        run_reference(args, ws, rank)
        return

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    gdr.load_library()
    pk, pk_kind = peaks()
    flush = l2_flusher(device)
    stream = torch.cuda.Stream(device=device)
    names = [w for w in args.workloads.split(",") if w]
    results = {}
    for i, name in enumerate(names):
        case = make_case(name, device, seed=rank)
        results[name] = bench_case(case, args, ws, rank, flush, stream, pk, pk_kind)
        del case
        torch.cuda.empty_cache()
    if ws == 1 and rank == 0 and not args.no_cpu_baseline:
        for name in names:
            if name in CPU_BASELINE_WORKLOADS:
                results[name]["cpu_baseline"] = cpu_baseline(name)

    if rank == 0:
        head = results[names[0]]
        line = {
            "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": head["dtype"], "data": "synthetic (seeded PCG64; see inputs.py)",
            "config": head["config"], "roofline": head["roofline"], "e2e": head["e2e"],
            "gpu_launches": head["gpu_launches"],
            # every workload's timed steps together (each line under
            # "workloads" carries its own count)
            "gpu_launches_all_workloads": sum(r["gpu_launches"] for r in results.values()),
            "clocks": head["clocks"],
        }
        if "cpu_baseline" in head:
            line["cpu_baseline"] = head["cpu_baseline"]
        line["workloads"] = {n: r for n, r in results.items() if n != names[0]}
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
