"""The debug build of the library (`build.py --debug`, -DSSD_DEBUG).

It compiles device-side checks into the tensor-core kernels: bounds of the global
stores and of the TMA coordinates, and barrier-phase checks (the B/C and x slots an
MMA reads hold the fill of that tile, and a product's completion is observed only
after the product was issued).  A failed check sets SSD_ERR_DEBUG_CHECK in the status
word and records the source line; nothing traps.  The CPU test builds it and checks
its exports; the GPU test runs small parity cases through it in a subprocess (the
binding loads the library SSD_B200_LIBRARY names) and expects no failed check and
results within the parity tolerance of the float64 oracle."""

import ctypes
import os
import subprocess
import sys

import pytest

from structured_state_space_chunked_b200 import build as ssd_build
from structured_state_space_chunked_b200 import ssd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_library_builds_and_reports_itself():
    path = ssd_build.build(debug=True)
    assert path.endswith("libssd_b200_debug.so") and os.path.exists(path)
    L = ctypes.CDLL(path)
    assert L.ssd_debug_build() == 1
    for name in ssd.ABI_SYMBOLS:
        assert hasattr(L, name), name
    assert ctypes.CDLL(ssd.library_path()).ssd_debug_build() == 0


_CHILD = r"""
import numpy as np, torch
from structured_state_space_chunked_b200 import inputs as I, ssd
from tests.parity_util import TOL, make, oracle_run, rel_err, to_np
assert ssd.lib().ssd_debug_build() == 1
cases = [
    # dtype, batch, seqlen, H, P, N, G, Q, init, varlen lengths
    ("bf16", 2, 300, 4, 64, 128, 1, 256, "normal0.1", None),   # N <= 128 kernel
    ("bf16", 1, 290, 2, 128, 256, 1, 256, "normal0.1", None),  # N = 256 kernel
    ("bf16", 1, 0, 4, 64, 128, 1, 128, "normal0.1", [1, 0, 300, 17, 129, 2]),
    ("fp32", 2, 200, 2, 32, 16, 1, 64, "zero", None),          # CUDA-core path
]
for dtype, b, L, H, P, N, G, Q, init, lens in cases:
    cu = None
    if lens is not None:
        cu = I.cu_seqlens_from_lengths(lens)
        L = int(cu[-1])
    w = I.random_small(50 + L, dtype, b, L, H, P, N, G, Q, init, varlen_tokens=L if lens else 0)
    inp = make(w, cu_seqlens=cu)
    bsz, Lr = inp["x"].shape[:2]
    nd = 0 if cu is None else len(lens)
    h = ssd.SSD(bsz, Lr, H, P, N, G, w.torch_dtype, max_docs=nd)
    y, fin = h.forward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], inp["dt_bias"],
                       Q, inp["initial_states"], inp["cu_seqlens"])
    st = h.status()
    line = h.debug_line()
    assert st == 0 and line == 0, (dtype, N, st, line)
    yr, fr = oracle_run(inp)
    ey, ef = rel_err(to_np(y), yr), rel_err(to_np(fin), fr)
    assert ey <= TOL[dtype] and ef <= TOL[dtype], (dtype, N, ey, ef)
    h.close()
print("debug-parity-ok")
"""


@pytest.mark.gpu
def test_debug_library_small_parity_and_no_failed_check():
    path = ssd_build.build(debug=True)
    env = dict(os.environ, SSD_B200_LIBRARY=path)
    r = subprocess.run([sys.executable, "-c", _CHILD], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and "debug-parity-ok" in r.stdout, r.stdout + r.stderr
