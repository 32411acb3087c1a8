"""ssd_forward_noalloc: the entry point for callers that may not allocate device
memory (for example applications that budget all device memory through their own
allocator, or code that cannot take the synchronisation an allocation may cause).
It takes no handle and keeps its scratch in a fixed 32 MiB array inside the
library.

The test calls it through the C ABI twice in a row (different problems, so the
second call runs on whatever the first left in the shared scratch) and checks
each output against the existing ssd_forward entry point and against the
float64 oracle, within the parity tolerance, then checks that a problem too big
for the array is refused.  This
file is collected last so that a stop-at-first-failure run has already run every
other test."""

import ctypes

import pytest
import torch

from structured_state_space_chunked_b200 import inputs as I
from structured_state_space_chunked_b200 import ssd
from tests.parity_util import TOL, make, oracle_run, rel_err, to_np

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(desc, inp, chunk, y, fin, status):
    ndocs = 0 if inp["cu_seqlens"] is None else inp["cu_seqlens"].numel() - 1
    return ssd.lib().ssd_forward_noalloc(
        ctypes.byref(desc), _p(inp["x"]), _p(inp["dt"]), _p(inp["A"]), _p(inp["B"]), _p(inp["C"]),
        _p(inp["D"]), _p(inp["dt_bias"]), int(chunk), _p(inp["initial_states"]),
        _p(inp["cu_seqlens"]), ndocs, _p(y), _p(fin), _p(status),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _reference(w, inp, chunk):
    ndocs = 0 if inp["cu_seqlens"] is None else inp["cu_seqlens"].numel() - 1
    bsz, L = inp["x"].shape[:2]
    h = ssd.SSD(bsz, L, w.nheads, w.headdim, w.dstate, w.ngroups, w.torch_dtype, max_docs=ndocs)
    y, fin = h.forward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                       inp["dt_bias"], chunk, inp["initial_states"], inp["cu_seqlens"])
    assert h.status() == 0
    return y, fin


def test_noalloc_matches_ssd_forward_on_two_calls_in_a_row():
    lens = [200, 1, 313, 0, 97]
    cu = I.cu_seqlens_from_lengths(lens)
    T = int(cu[-1])
    problems = [
        (I.random_small(31, "fp32", 2, 300, 4, 32, 64, 2, 64, "normal0.1"), None),
        (I.random_small(32, "bf16", 1, T, 4, 64, 128, 1, 128, "normal0.1", varlen_tokens=T), cu),
    ]
    status = torch.full((1,), 123, dtype=torch.int32, device="cuda")
    for w, cus in problems:
        inp = make(w, cu_seqlens=cus)
        bsz, L = inp["x"].shape[:2]
        ndocs = len(lens) if cus is not None else bsz
        desc = ssd.make_desc(bsz, L, w.nheads, w.headdim, w.dstate, w.ngroups, w.torch_dtype,
                             max_docs=ndocs if cus is not None else 0)
        y = torch.empty_like(inp["x"])
        fin = torch.empty(ndocs, w.nheads, w.dstate, w.headdim, device="cuda")
        rc = _noalloc(desc, inp, w.chunk_size, y, fin, status)
        assert rc == 0, ssd.ERRORS.get(rc, rc)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        y_ref, fin_ref = _reference(w, inp, w.chunk_size)
        tol = TOL[w.dtype]
        assert rel_err(to_np(y), to_np(y_ref)) <= tol
        assert rel_err(to_np(fin), to_np(fin_ref)) <= tol
        # and directly against the float64 oracle on the same inputs
        y_or, fin_or = oracle_run(inp)
        assert rel_err(to_np(y), y_or) <= tol
        assert rel_err(to_np(fin), fin_or) <= tol


def test_noalloc_refuses_a_problem_larger_than_its_scratch():
    # fp32, 4096 tokens, 16 heads, N x P = 128 x 64, Q = 64: the chunk states alone
    # need 64 * 16 * 128 * 64 * 4 bytes = 32 MiB, more than the array holds
    w = I.random_small(33, "fp32", 1, 4096, 16, 64, 128, 1, 64)
    inp = make(w)
    desc = ssd.make_desc(1, 4096, 16, 64, 128, 1, torch.float32)
    y = torch.full_like(inp["x"], 5.0)
    fin = torch.empty(1, 16, 128, 64, device="cuda")
    rc = _noalloc(desc, inp, 64, y, fin, None)
    assert rc == -7, ssd.ERRORS.get(rc, rc)
    torch.cuda.synchronize()
    assert torch.all(y == 5.0)
