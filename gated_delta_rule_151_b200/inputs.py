"""Seeded synthetic inputs for the gated delta-rule recurrence.

This module is the one piece shared by the CUDA path's callers and the
oracle's callers.  It holds none of the recurrence's arithmetic: it only
draws random numbers, applies the input-side maps the workloads describe
(L2 normalisation of q and k, a sigmoid for the write strength beta, and
``g = -softplus(x) * c`` for the log-gate), and rounds once to the I/O
precision.

Recipe (every workload, both sides):

* Draws are standard normals in float64 from numpy's PCG64.  Tensor ``X``
  (one of ``q, k, v, beta, gate, h0`` -- ids 0..5, cut points id 6) is cut
  along its leading axis into fixed blocks of ``BLOCK_ELEMS`` elements; block
  ``b`` draws from ``SeedSequence(seed, spawn_key=(id, b))``.  The values
  therefore do not depend on how many threads generate them.
* q, k: N(0, 1) per element, then divided by their L2 norm over d_k per
  (token, head), in float64.
* v: N(0, 1).
* beta = sigmoid(x), x ~ N(0, 1).
* log-gate g = -softplus(x) * c, x ~ N(0, 1); shape [T, H] (scalar gate,
  Gated DeltaNet) or [T, H, d_k] (channel gate, Kimi Delta Attention).
* h0 ~ N(0, std^2) per element when the workload has a nonzero initial state.
* Rounding: q, k, v go float64 -> float32 (round to nearest even) and, for
  bf16 I/O, float32 -> bfloat16 (round to nearest even, torch's conversion);
  beta, g and h0 go to float32.
* Variable-length packing: 7 distinct cut points drawn uniformly from
  [1, total_T - 1] (rejecting repeats), sorted; cu_seqlens = [0, cuts, total_T].

Workloads (the page on the Flash model architectures, section "Linear
attention: a fixed-size memory in place of the cache", gives the two update
rules; the shapes are the benchmark set of this library):

=================  ==========================================================
tiny_gdn           1 sequence, H=2, T=64, d=16, fp32 I/O, c=0.1, h0=0
gdn_prefill        1 sequence, H=16, T=8192, d=128, bf16, scalar gate c=0.05
kda_prefill        2 sequences x 32768, H=32, d=128, bf16, channel gate
                   c=0.05, h0 ~ N(0, 0.02^2)
decode_gdn/kda     256 sequences, H=32, d=128, 512 steps of one bf16 token,
                   c=0.1, h0 ~ N(0, 0.02^2) (state 512 MiB fp32)
decode_spec_gdn    the decode_gdn tokens verified 4 at a time (128 steps of
                   4 draft tokens per sequence)
backward_gdn       the gdn_prefill inputs with upstream gradients dO ~ N(0, 1)
                   (bf16) and dS_final ~ N(0, 1) for the gradient
prologue_gdn       raw prologue inputs at the gdn_prefill shape (1 x 8192
                   tokens, H=16, d=128, bf16): x_q, x_k, x_v ~ N(0, 1), taps
                   ~ N(0, 0.5^2), convolution state ~ N(0, 1), x_g, x_beta
                   ~ N(0, 1), gate coefficient c=0.05 per head
varlen_gdn         8 packed sequences, 262144 tokens, H=16, d=128, bf16,
                   scalar gate c=0.1, h0=0
gqa_prefill        1 sequence, 8192 tokens, 16 query/key heads shared by 48
                   value heads (3 each), d=128, bf16, scalar gate c=0.05
prefill_fused_gdn  the prologue_gdn raw inputs through the prologue fused into
                   the chunked prefill (o and the final state out)
kda_prefill_small  kda_prefill at 2 x 2048 tokens (the same 64 chains and
                   plan at a sixteenth of the length; a profiler capture
                   holds a few hundred MB on the device instead of 7 GB)
=================  ==========================================================

With grouped heads (``H_qk`` < ``H``), q and k carry ``H_qk`` heads and value
head h reads query/key head ``h // (H // H_qk)``.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np
import torch

BLOCK_ELEMS = 1 << 21

_ID = {"q": 0, "k": 1, "v": 2, "beta": 3, "gate": 4, "h0": 5, "cuts": 6,
       # raw inputs of the prologue (before the convolution and the maps)
       "xq": 7, "xk": 8, "xv": 9, "wq": 10, "wk": 11, "wv": 12, "xg": 13, "xb": 14,
       "conv": 15,
       # upstream gradients of the backward pass
       "do": 16, "dsf": 17}

SCALAR = "scalar"    # Gated DeltaNet: one gate per head and token
CHANNEL = "channel"  # Kimi Delta Attention: one gate per key channel


def _threads() -> int:
    try:
        return max(1, min(16, len(os.sched_getaffinity(0))))
    except AttributeError:  # pragma: no cover
        return max(1, min(16, os.cpu_count() or 1))


def _blocks(shape):
    inner = int(np.prod(shape[1:], dtype=np.int64)) if len(shape) > 1 else 1
    rows = max(1, BLOCK_ELEMS // max(inner, 1))
    n0 = shape[0]
    return [(b, r0, min(n0, r0 + rows)) for b, r0 in enumerate(range(0, n0, rows))]


def _fill(seed: int, name: str, shape, fn, out_dtype) -> np.ndarray:
    """Draw N(0,1) float64 blocks for tensor `name`, map each block with `fn`
    (float64 -> float64) and store it rounded to `out_dtype`."""
    out = np.empty(shape, dtype=out_dtype)
    if out.size == 0:
        return out
    tid = _ID[name]

    def work(blk):
        b, r0, r1 = blk
        rng = np.random.default_rng(np.random.SeedSequence(seed, spawn_key=(tid, b)))
        x = rng.standard_normal((r1 - r0,) + tuple(shape[1:]))
        out[r0:r1] = fn(x).astype(out_dtype)

    blocks = _blocks(shape)
    if len(blocks) == 1:
        work(blocks[0])
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, blocks))
    return out


def _l2norm(x: np.ndarray) -> np.ndarray:
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True))


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


def _softplus(x: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, x)


@dataclass
class Inputs:
    """One workload's rounded inputs as CPU torch tensors.

    q, k: [total_T, H_qk, d_k]; v: [total_T, H, d_v] in ``io_dtype``;
    g: [total_T, H] (scalar) or [total_T, H, d_k] (channel) float32;
    beta: [total_T, H] float32; h0: [num_seqs, H, d_v, d_k] float32 or None;
    cu_seqlens: int32 [num_seqs + 1] (always filled in, also for equal
    lengths).
    """

    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor
    beta: torch.Tensor
    h0: torch.Tensor | None
    cu_seqlens: torch.Tensor
    gate_mode: str
    io_dtype: torch.dtype
    meta: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return int(self.cu_seqlens.numel() - 1)

    @property
    def total_T(self) -> int:
        return int(self.q.shape[0])

    @property
    def H(self) -> int:
        return int(self.v.shape[1])

    @property
    def H_qk(self) -> int:
        return int(self.q.shape[1])

    @property
    def d_k(self) -> int:
        return int(self.q.shape[2])

    @property
    def d_v(self) -> int:
        return int(self.v.shape[2])

    def equal_lengths(self) -> bool:
        cu = self.cu_seqlens.tolist()
        n = len(cu) - 1
        return n > 0 and self.total_T % n == 0 and all(
            cu[i] == i * (self.total_T // n) for i in range(n + 1))


def random_cu_seqlens(seed: int, total_T: int, num_seqs: int) -> np.ndarray:
    """num_seqs-1 distinct cut points uniform on [1, total_T-1], sorted."""
    if num_seqs < 1:
        raise ValueError("num_seqs must be >= 1")
    if num_seqs - 1 > max(total_T - 1, 0):
        raise ValueError("more sequences than tokens")
    rng = np.random.default_rng(np.random.SeedSequence(seed, spawn_key=(_ID["cuts"], 0)))
    cuts: list[int] = []
    while len(cuts) < num_seqs - 1:
        c = int(rng.integers(1, total_T))  # [1, total_T-1]
        if c not in cuts:
            cuts.append(c)
    return np.array([0] + sorted(cuts) + [total_T], dtype=np.int32)


def make_inputs(*, total_T: int, H: int, d_k: int, d_v: int | None = None,
                H_qk: int | None = None,
                num_seqs: int = 1, cu_seqlens=None, gate_mode: str = SCALAR,
                io_dtype: torch.dtype = torch.bfloat16, c: float = 0.05,
                h0_std: float = 0.0, seed: int = 0, meta: dict | None = None) -> Inputs:
    """Draw one workload following the module recipe.

    ``cu_seqlens`` may be given explicitly (any non-decreasing int sequence
    from 0 to total_T); otherwise ``num_seqs`` equal sequences are used.
    """
    d_v = d_k if d_v is None else d_v
    H_qk = H if H_qk is None else H_qk
    if H_qk < 1 or H % H_qk:
        raise ValueError("H_qk must divide H")
    if gate_mode not in (SCALAR, CHANNEL):
        raise ValueError(f"gate_mode {gate_mode!r}")
    if io_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("io_dtype must be bfloat16 or float32")
    if cu_seqlens is None:
        if num_seqs < 1 or total_T % num_seqs:
            raise ValueError("total_T must divide into num_seqs equal sequences")
        cu = np.arange(num_seqs + 1, dtype=np.int64) * (total_T // num_seqs)
    else:
        cu = np.asarray(cu_seqlens, dtype=np.int64)
        num_seqs = len(cu) - 1
        if cu[0] != 0 or cu[-1] != total_T or np.any(np.diff(cu) < 0):
            raise ValueError("cu_seqlens must run from 0 to total_T, non-decreasing")

    q = _fill(seed, "q", (total_T, H_qk, d_k), _l2norm, np.float32)
    k = _fill(seed, "k", (total_T, H_qk, d_k), _l2norm, np.float32)
    v = _fill(seed, "v", (total_T, H, d_v), lambda x: x, np.float32)
    beta = _fill(seed, "beta", (total_T, H), _sigmoid, np.float32)
    gshape = (total_T, H) if gate_mode == SCALAR else (total_T, H, d_k)
    g = _fill(seed, "gate", gshape, lambda x: -_softplus(x) * c, np.float32)
    h0 = None
    if h0_std > 0.0:
        h0 = torch.from_numpy(_fill(seed, "h0", (num_seqs, H, d_v, d_k),
                                    lambda x: x * h0_std, np.float32))

    def io(a):
        t = torch.from_numpy(a)
        return t.to(io_dtype) if io_dtype != torch.float32 else t

    m = {"seed": seed, "c": c, "h0_std": h0_std, "gate_mode": gate_mode,
         "io_dtype": str(io_dtype).replace("torch.", "")}
    if meta:
        m.update(meta)
    return Inputs(q=io(q), k=io(k), v=io(v), g=torch.from_numpy(g),
                  beta=torch.from_numpy(beta), h0=h0,
                  cu_seqlens=torch.from_numpy(cu.astype(np.int32)),
                  gate_mode=gate_mode, io_dtype=io_dtype, meta=m)


@dataclass
class PrologueInputs:
    """Raw inputs of the input-side prologue as CPU torch tensors.

    xq, xk: [total_T, H_qk, d_k]; xv: [total_T, H, d_v] in ``io_dtype``;
    wq, wk: [H_qk d_k, 4]; wv: [H d_v, 4] float32 taps (tap 3 takes the current
    token); xg: [total_T, H] or [total_T, H, d_k] and xb: [total_T, H] float32;
    gscale: [H] float32; conv_state: [num_seqs, 2 H_qk d_k + H d_v, 3]
    float32 or None; cu_seqlens: int32 [num_seqs + 1].
    """

    xq: torch.Tensor
    xk: torch.Tensor
    xv: torch.Tensor
    wq: torch.Tensor
    wk: torch.Tensor
    wv: torch.Tensor
    xg: torch.Tensor
    gscale: torch.Tensor
    xb: torch.Tensor
    conv_state: torch.Tensor | None
    cu_seqlens: torch.Tensor
    gate_mode: str
    io_dtype: torch.dtype
    meta: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return int(self.cu_seqlens.numel() - 1)

    @property
    def total_T(self) -> int:
        return int(self.xq.shape[0])

    @property
    def H(self) -> int:
        return int(self.xv.shape[1])

    @property
    def H_qk(self) -> int:
        return int(self.xq.shape[1])

    @property
    def d_k(self) -> int:
        return int(self.xq.shape[2])

    @property
    def d_v(self) -> int:
        return int(self.xv.shape[2])

    @property
    def h0(self):
        return None


def make_prologue_inputs(*, total_T: int, H: int, d_k: int, d_v: int | None = None,
                         H_qk: int | None = None, num_seqs: int = 1, cu_seqlens=None,
                         gate_mode: str = SCALAR, io_dtype: torch.dtype = torch.bfloat16,
                         c: float = 0.05, tap_std: float = 0.5, state_std: float = 1.0,
                         seed: int = 0, meta: dict | None = None) -> PrologueInputs:
    """Draw raw prologue inputs: standard normals (taps and state scaled by
    their standard deviations), rounded once to the I/O precision."""
    d_v = d_k if d_v is None else d_v
    H_qk = H if H_qk is None else H_qk
    if H_qk < 1 or H % H_qk:
        raise ValueError("H_qk must divide H")
    if cu_seqlens is None:
        if num_seqs < 1 or total_T % num_seqs:
            raise ValueError("total_T must divide into num_seqs equal sequences")
        cu = np.arange(num_seqs + 1, dtype=np.int64) * (total_T // num_seqs)
    else:
        cu = np.asarray(cu_seqlens, dtype=np.int64)
        num_seqs = len(cu) - 1
        if cu[0] != 0 or cu[-1] != total_T or np.any(np.diff(cu) < 0):
            raise ValueError("cu_seqlens must run from 0 to total_T, non-decreasing")
    ident = lambda x: x  # noqa: E731
    xq = _fill(seed, "xq", (total_T, H_qk, d_k), ident, np.float32)
    xk = _fill(seed, "xk", (total_T, H_qk, d_k), ident, np.float32)
    xv = _fill(seed, "xv", (total_T, H, d_v), ident, np.float32)
    taps = lambda x: x * tap_std  # noqa: E731
    wq = _fill(seed, "wq", (H_qk * d_k, 4), taps, np.float32)
    wk = _fill(seed, "wk", (H_qk * d_k, 4), taps, np.float32)
    wv = _fill(seed, "wv", (H * d_v, 4), taps, np.float32)
    gshape = (total_T, H) if gate_mode == SCALAR else (total_T, H, d_k)
    xg = _fill(seed, "xg", gshape, ident, np.float32)
    xb = _fill(seed, "xb", (total_T, H), ident, np.float32)
    conv = None
    if state_std > 0.0:
        conv = torch.from_numpy(_fill(seed, "conv", (num_seqs, 2 * H_qk * d_k + H * d_v, 3),
                                      lambda x: x * state_std, np.float32))

    def io(a):
        t = torch.from_numpy(a)
        return t.to(io_dtype) if io_dtype != torch.float32 else t

    m = {"seed": seed, "c": c, "tap_std": tap_std, "state_std": state_std,
         "gate_mode": gate_mode, "io_dtype": str(io_dtype).replace("torch.", "")}
    if meta:
        m.update(meta)
    return PrologueInputs(xq=io(xq), xk=io(xk), xv=io(xv), wq=torch.from_numpy(wq),
                          wk=torch.from_numpy(wk), wv=torch.from_numpy(wv),
                          xg=torch.from_numpy(xg), gscale=torch.full((H,), c, dtype=torch.float32),
                          xb=torch.from_numpy(xb), conv_state=conv,
                          cu_seqlens=torch.from_numpy(cu.astype(np.int32)),
                          gate_mode=gate_mode, io_dtype=io_dtype, meta=m)


# ---------------------------------------------------------------------------
# The benchmark workloads.
# ---------------------------------------------------------------------------

WORKLOADS = ("tiny_gdn", "gdn_prefill", "kda_prefill", "decode_gdn",
             "decode_kda", "varlen_gdn", "gqa_prefill", "decode_spec_gdn", "prologue_gdn",
             "backward_gdn", "kda_prefill_small", "prefill_fused_gdn")

SPEC_DRAFT = 4   # tokens verified per sequence per step in decode_spec_gdn

DECODE_SEQS, DECODE_HEADS, DECODE_D, DECODE_STEPS = 256, 32, 128, 512


def workload(name: str, seed: int = 0) -> Inputs:
    """The named benchmark workload (module docstring table).

    Decode workloads come packed like a prefill over the 512 steps of each
    sequence (token-major per sequence); ``decode_view`` reshapes them to the
    per-step layout [steps, N, H, d] a decode loop consumes.
    """
    if name == "tiny_gdn":
        return make_inputs(total_T=64, H=2, d_k=16, num_seqs=1, gate_mode=SCALAR,
                           io_dtype=torch.float32, c=0.1, seed=seed,
                           meta={"workload": name})
    if name == "gdn_prefill":
        return make_inputs(total_T=8192, H=16, d_k=128, num_seqs=1, gate_mode=SCALAR,
                           io_dtype=torch.bfloat16, c=0.05, seed=seed,
                           meta={"workload": name})
    if name in ("kda_prefill", "kda_prefill_small"):
        T = 65536 if name == "kda_prefill" else 4096
        return make_inputs(total_T=T, H=32, d_k=128, num_seqs=2, gate_mode=CHANNEL,
                           io_dtype=torch.bfloat16, c=0.05, h0_std=0.02, seed=seed,
                           meta={"workload": name})
    if name in ("decode_gdn", "decode_kda", "decode_spec_gdn"):
        mode = CHANNEL if name == "decode_kda" else SCALAR
        return make_inputs(total_T=DECODE_SEQS * DECODE_STEPS, H=DECODE_HEADS,
                           d_k=DECODE_D, num_seqs=DECODE_SEQS, gate_mode=mode,
                           io_dtype=torch.bfloat16, c=0.1, h0_std=0.02, seed=seed,
                           meta={"workload": name, "steps": DECODE_STEPS})
    if name == "gqa_prefill":
        return make_inputs(total_T=8192, H=48, H_qk=16, d_k=128, num_seqs=1,
                           gate_mode=SCALAR, io_dtype=torch.bfloat16, c=0.05, seed=seed,
                           meta={"workload": name})
    if name == "varlen_gdn":
        cu = random_cu_seqlens(seed, 262144, 8)
        return make_inputs(total_T=262144, H=16, d_k=128, cu_seqlens=cu,
                           gate_mode=SCALAR, io_dtype=torch.bfloat16, c=0.1,
                           seed=seed, meta={"workload": name})
    raise KeyError(name)


def make_grad_inputs(inp: Inputs, seed: int = 0, dsf_std: float = 1.0):
    """Upstream gradients for the backward pass of ``inp``: dO [total_T, H,
    d_v] ~ N(0, 1) rounded to the I/O type, and dS_final [num_seqs, H, d_v,
    d_k] ~ N(0, dsf_std^2) in float32 (None when dsf_std is 0)."""
    dO = _fill(seed, "do", (inp.total_T, inp.H, inp.d_v), lambda x: x, np.float32)
    dO = torch.from_numpy(dO)
    if inp.io_dtype != torch.float32:
        dO = dO.to(inp.io_dtype)
    dsf = None
    if dsf_std > 0.0:
        dsf = torch.from_numpy(_fill(seed, "dsf", (inp.num_seqs, inp.H, inp.d_v, inp.d_k),
                                     lambda x: x * dsf_std, np.float32))
    return dO, dsf


def prologue_workload(name: str = "prologue_gdn", seed: int = 0) -> PrologueInputs:
    """Raw prologue inputs at the gdn_prefill shape (module docstring table);
    the fused prefill workload takes the same inputs."""
    if name not in ("prologue_gdn", "prefill_fused_gdn"):
        raise KeyError(name)
    return make_prologue_inputs(total_T=8192, H=16, d_k=128, num_seqs=1, gate_mode=SCALAR,
                                io_dtype=torch.bfloat16, c=0.05, tap_std=0.5, state_std=1.0,
                                seed=seed, meta={"workload": name})


def decode_view(x: torch.Tensor, num_seqs: int) -> torch.Tensor:
    """[N*steps, ...] sequence-major -> [steps, N, ...] step-major (a copy)."""
    steps = x.shape[0] // num_seqs
    return x.reshape(num_seqs, steps, *x.shape[1:]).transpose(0, 1).contiguous()
