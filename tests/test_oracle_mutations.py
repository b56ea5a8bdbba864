"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a private copy of the oracle's C source
(never in the real one), compiles it with gcc into a temporary library, and
checks that the independent pins -- the hand-worked examples and the
transition-matrix expansion -- reject it.  CPU only.
"""
import ctypes
import json
import os
import subprocess
import tempfile

import numpy as np
import pytest

from oracle import brute_force
from oracle.loop import _SRC

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")

MUTATIONS = {
    "erase_uses_undecayed_state": ("x += S[r * dk + j] * kt[j];",
                                   "x += S[r * dk + j] * kt[j] / a[j];"),
    "output_reads_pre_write_state": ("y += S[r * dk + j] * qt[j];",
                                     "y += (S[r * dk + j] - u[r] * kt[j]) * qt[j];"),
    "gate_on_value_channels": ("S[r * dk + j] *= a[j];", "S[r * dk + j] *= a[r % dk];"),
    "erase_sign_flipped": ("u[r] = bt * (vt[r] - x);", "u[r] = bt * (vt[r] + x);"),
    "write_strength_dropped": ("u[r] = bt * (vt[r] - x);", "u[r] = (vt[r] - x);"),
    "state_transposed": ("x += S[r * dk + j] * kt[j];", "x += S[j * dk + r] * kt[j];"),
    "key_for_query": ("y += S[r * dk + j] * qt[j];", "y += S[r * dk + j] * kt[j];"),
}


def _compile(src_text, tmpdir, name):
    c = os.path.join(tmpdir, name + ".c")
    so = os.path.join(tmpdir, name + ".so")
    open(c, "w").write(src_text)
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-o", so, c,
                           "-lpthread", "-lm"])
    lib = ctypes.CDLL(so)
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    lib.gdr_oracle_run.argtypes = [P, P, P, P, P, P, P, I64, I64, I64, I64, I64, ctypes.c_int,
                                   P, P, ctypes.c_int]
    lib.gdr_oracle_run.restype = ctypes.c_int
    return lib


def _run(lib, q, k, v, g, beta, S0, channel):
    arr = lambda x: np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    q, k, v, g, beta, S0 = map(arr, (q, k, v, g, beta, S0))
    T, dk = k.shape
    dv = v.shape[1]
    cu = np.array([0, T], dtype=np.int64)
    o = np.empty((T, dv))
    fin = np.empty((dv, dk))
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    rc = lib.gdr_oracle_run(p(q), p(k), p(v), p(g), p(beta), p(S0), p(cu), 1, 1, 1, dk, dv,
                            int(channel), p(o), p(fin), 1)
    assert rc == 0
    return o, fin


def _pins_pass(lib):
    """True when the library passes every pin used here."""
    for ex in json.load(open(GOLDEN))["examples"]:
        ch = ex["gate_mode"] == "channel"
        o, S = _run(lib, ex["q"], ex["k"], ex["v"], np.log(np.asarray(ex["alpha"], float)),
                    ex["beta"], ex["S0"], ch)
        if not (np.allclose(o, ex["expect_o"], atol=1e-9) and np.allclose(S, ex["expect_S"], atol=1e-9)):
            return False
    rng = np.random.default_rng(3)
    T, d = 6, 8
    for ch in (False, True):
        q = rng.standard_normal((T, d)); q /= np.linalg.norm(q, axis=1, keepdims=True)
        k = rng.standard_normal((T, d)); k /= np.linalg.norm(k, axis=1, keepdims=True)
        v = rng.standard_normal((T, d))
        beta = 1 / (1 + np.exp(-rng.standard_normal(T)))
        g = -np.logaddexp(0, rng.standard_normal((T, d) if ch else T)) * 0.5
        S0 = rng.standard_normal((d, d))
        o, S = _run(lib, q, k, v, g, beta, S0, ch)
        eo, st = brute_force.expand(q, k, v, np.exp(g), beta, S0)
        if not (np.allclose(o, eo, atol=1e-10) and np.allclose(S, st[-1], atol=1e-10)):
            return False
    return True


@pytest.fixture(scope="module")
def tmpdir():
    with tempfile.TemporaryDirectory() as d:
        yield d


def test_unmodified_source_passes(tmpdir):
    assert _pins_pass(_compile(open(_SRC).read(), tmpdir, "orig"))


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tmpdir, name):
    old, new = MUTATIONS[name]
    src = open(_SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    lib = _compile(src.replace(old, new), tmpdir, name)
    assert not _pins_pass(lib), f"pins did not catch: {name}"
