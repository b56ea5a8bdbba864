"""gated_delta_rule_151_b200 -- the gated delta-rule recurrence on NVIDIA B200.

``gdr`` is the ctypes binding of libgdr.so (include/gdr.h): chunked prefill
and single-token decode in scalar-gate (Gated DeltaNet) and channel-gate
(Kimi Delta Attention) modes.  ``inputs`` draws the seeded synthetic
workloads.  Importing the package loads nothing; the library is loaded on the
first call and every call raises if it is missing.
"""
from . import gdr  # noqa: F401
from .gdr import (GdrError, gdr_decode_multi, gdr_decode_step, gdr_decode_step_gqa,  # noqa: F401
                  gdr_prefill_check_workspace, gdr_prefill_chunked, gdr_prefill_chunked_gqa,
                  gdr_prefill_chunked_noalloc, gdr_prefill_path, gdr_prefill_workspace_size,
                  gdr_status_string, load_library)
