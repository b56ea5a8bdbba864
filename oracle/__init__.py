"""fp64 CPU oracle for the gated delta-rule recurrence.

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the
benchmark's CPU-baseline leg are the only callers.  Nothing here is imported by
the CUDA path, and nothing here imports it.

* ``run``         -- the sequential token loop (plain C, fp64, one POSIX thread
                     per core over independent (sequence, head) pairs).
* ``brute_force`` -- an independent expansion of the recurrence into explicit
                     d_k x d_k transition matrices, used to pin the loop.
* ``backward``    -- the gradient of the recurrence (reverse token sweep, numpy
                     float64), pinned by finite differences of ``run``.
* ``prologue``    -- the input-side prologue (short causal convolution with its
                     state, q/k L2 normalisation, gate and beta maps) in numpy
                     float64.

Both follow the page "How the New Flash Models Work: Inside GLM-5.3-Flash and
Qwen3.8-Flash-Next", section "Linear attention: a fixed-size memory in place of
the cache" (Gated DeltaNet and Kimi Delta Attention equations).
"""
from .loop import run, build, library_path  # noqa: F401
from . import brute_force  # noqa: F401
from . import prologue  # noqa: F401
from . import backward  # noqa: F401
