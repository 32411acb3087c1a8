"""GPU parity of ssd_backward against the float64 backward oracle.

The oracle is the chain rule taken backwards through the sequential recurrence
("Transformers are SSMs", paperlayer.ai summary, §3.4.1), pinned by finite
differences and autograd in test_oracle_pins.py.  The CUDA path differentiates the
block decomposition of §6 in fp32.  Both sides see the same (device-rounded) inputs.

Tolerance (max |err| / max |ref|).  fp32 inputs (CUDA cores, fp32 throughout): 1e-4
for the per-token gradients and the initial-state gradient, as for the forward's fp32
outputs; 1e-3 for dA, dD and dt_bias, each a sum over every token of the head whose
terms cancel (the sum can be much smaller than its largest terms, and fp32 atomics add
them in any order).  bf16 inputs: 2e-2 for every gradient, as for the forward's bf16
path -- with P a multiple of 64 and N = 64 or 128 the in-chunk products run on the
tensor cores with bf16 operands (the weighted matrices W' and V and the states rounded
to bf16), one block per 64-column slice of P whose parts of every sum over p add up in
the gradients.
"""

import numpy as np
import pytest
import torch

import oracle
from structured_state_space_chunked_b200 import inputs as I
from structured_state_space_chunked_b200 import ssd
from tests.parity_util import make, rel_err, to_np

pytestmark = pytest.mark.gpu

TOK_TOL = 1e-4
SUM_TOL = 1e-3
BF16_TOL = 2e-2


def _tols(dtype):
    return (BF16_TOL, BF16_TOL) if dtype == "bf16" else (TOK_TOL, SUM_TOL)
PER_TOKEN = ("dx", "ddt", "dB", "dC", "dinitial_states")
PER_HEAD = ("dA", "dD", "ddt_bias")


def _run(w, inp, dy, dfin, handle=None):
    max_docs = 0 if inp["cu_seqlens"] is None else inp["cu_seqlens"].numel() - 1
    bsz, L = inp["x"].shape[:2]
    h = handle or ssd.SSD(bsz, L, w.nheads, w.headdim, w.dstate, w.ngroups, w.torch_dtype,
                          max_docs=max_docs)
    g = h.backward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], dy, inp["D"],
                   inp["dt_bias"], inp["initial_states"], dfin, inp["cu_seqlens"])
    assert h.status() == 0
    torch.cuda.synchronize()
    return {k: to_np(v) for k, v in g.items()}


def _oracle(inp, dy, dfin, heads=None, nthreads=0):
    cpu = lambda t: None if t is None else t.cpu()  # noqa: E731
    cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].cpu().numpy()
    return oracle.oracle_backward(cpu(inp["x"]), cpu(inp["dt"]), cpu(inp["A"]), cpu(inp["B"]),
                                  cpu(inp["C"]), cpu(dy), cpu(inp["D"]), cpu(inp["dt_bias"]),
                                  cpu(inp["initial_states"]), cpu(dfin), cu_seqlens=cu,
                                  heads=heads, nthreads=nthreads)


SMALL = [
    # dtype, batch, seqlen, H, P, N, G, init, varlen tokens
    ("fp32", 2, 300, 4, 64, 128, 2, "normal0.1", 0),
    ("bf16", 2, 300, 4, 64, 128, 1, "normal0.1", 0),
    ("fp32", 1, 200, 3, 16, 16, 1, "zero", 0),
    ("fp32", 1, 130, 2, 80, 72, 2, "normal0.1", 0),
    ("fp32", 1, 64, 2, 128, 256, 1, "normal0.1", 0),
    ("bf16", 1, 0, 4, 64, 64, 2, "normal0.1", 1500),
    ("fp32", 3, 1, 2, 32, 32, 1, "normal0.1", 0),
    ("bf16", 2, 700, 4, 64, 128, 2, "normal0.1", 0),
    ("bf16", 1, 300, 2, 32, 64, 1, "normal0.1", 0),
    ("bf16", 1, 0, 4, 64, 128, 1, "normal0.1", 3000),
    ("bf16", 2, 300, 4, 128, 128, 2, "normal0.1", 0),
    ("bf16", 1, 0, 4, 128, 64, 2, "normal0.1", 1500),
    ("bf16", 1, 270, 2, 192, 128, 1, "normal0.1", 0),
]


@pytest.mark.parametrize("case", SMALL, ids=["fp32-G2", "bf16", "tiny-P16N16", "ragged-P80N72",
                                              "one-chunk-N256", "bf16-packed", "one-token",
                                              "bf16-G2-L700", "bf16-P32-cudacores",
                                              "bf16-packed-N128", "bf16-P128-tc", "bf16-P128-N64-packed",
                                              "bf16-P192-tc"])
def test_backward_matches_oracle(case):
    dtype, b, L, H, P, N, G, init, vt = case
    w = I.random_small(300 + P + N + L, dtype, b, L, H, P, N, G, 64, init, vt)
    inp = make(w)
    ndocs = b if inp["cu_seqlens"] is None else inp["cu_seqlens"].numel() - 1
    dy, dfin = I.make_cotangents(w, ndocs, device="cuda")
    got = _run(w, inp, dy, dfin)
    ref = _oracle(inp, dy, dfin)
    tok_tol, sum_tol = _tols(dtype)
    for k in PER_TOKEN:
        e = rel_err(got[k], ref[k])
        assert e <= tok_tol, f"{k} rel err {e:.3e}"
    for k in PER_HEAD:
        e = rel_err(got[k], ref[k])
        assert e <= sum_tol, f"{k} rel err {e:.3e}"


def test_backward_packed_documents_with_an_empty_one():
    w = I.random_small(77, "fp32", 1, 0, 2, 32, 64, 1, 64, "normal0.1", 700)
    cu = np.array([0, 100, 100, 389, 700], dtype=np.int32)
    inp = make(w, cu_seqlens=cu)
    dy, dfin = I.make_cotangents(w, 4, device="cuda")
    got = _run(w, inp, dy, dfin)
    ref = _oracle(inp, dy, dfin)
    for k in PER_TOKEN:
        assert rel_err(got[k], ref[k]) <= TOK_TOL, k
    for k in PER_HEAD:
        assert rel_err(got[k], ref[k]) <= SUM_TOL, k
    # the empty document passes its final-state cotangent straight through
    assert np.array_equal(got["dinitial_states"][1], to_np(dfin)[1])


def test_only_final_state_cotangent_gives_the_pure_decay():
    """dy = 0: the initial-state gradient is exp(sum of delta A over the document)
    times dfinal, and dx, dB, dC see only the final state."""
    w = I.random_small(5, "fp32", 2, 333, 3, 64, 64, 1, 64, "normal0.1")
    inp = make(w)
    dy = torch.zeros(2, 333, 3, 64, device="cuda")
    _, dfin = I.make_cotangents(w, 2, device="cuda")
    got = _run(w, inp, dy, dfin)
    delta = torch.nn.functional.softplus(inp["dt"].double() + inp["dt_bias"].double())
    total = (delta * inp["A"].double()).sum(dim=1)                      # [b, H]
    expect = torch.exp(total)[:, :, None, None] * dfin.double()
    assert rel_err(got["dinitial_states"], to_np(expect)) <= TOK_TOL
    assert np.all(got["dD"] == 0)


@pytest.mark.parametrize("name,heads", [("mamba2_130m_layer_b4_L2048", [0, 13, 23]),
                                        ("mamba2_2p7b_layer_b8_L4096", [5, 79]),
                                        ("long_L16384_H64_P128_N128_G8", [0, 37, 63])])
def test_backward_full_size_sampled_heads(name, heads):
    w = I.workload(name)
    inp = make(w)
    ndocs = w.batch
    dy, dfin = I.make_cotangents(w, ndocs, device="cuda")
    got = _run(w, inp, dy, dfin)
    ref = _oracle(inp, dy, dfin, heads=heads, nthreads=4)
    tok_tol, sum_tol = _tols(w.dtype)
    for k in ("dx", "ddt"):
        e = rel_err(got[k][:, :, heads], ref[k][:, :, heads])
        assert e <= tok_tol, f"{k} rel err {e:.3e}"
    e = rel_err(got["dinitial_states"][:, heads], ref["dinitial_states"][:, heads])
    assert e <= tok_tol, f"dinitial_states rel err {e:.3e}"
    for k in PER_HEAD:
        e = rel_err(got[k][heads], ref[k][heads])
        assert e <= sum_tol, f"{k} rel err {e:.3e}"
    # dD is sum <dy, x> over the head's tokens, for every head
    dD = (dy.double() * inp["x"].double()).sum(dim=(0, 1, 3))
    assert rel_err(got["dD"], to_np(dD)) <= sum_tol


def test_backward_wide_head_dim():
    w = I.random_small(41, "fp32", 1, 150, 2, 256, 64, 1, 64, "normal0.1")
    inp = make(w)
    dy, dfin = I.make_cotangents(w, 1, device="cuda")
    got = _run(w, inp, dy, dfin)
    ref = _oracle(inp, dy, dfin)
    for k in PER_TOKEN:
        assert rel_err(got[k], ref[k]) <= TOK_TOL, k
    for k in PER_HEAD:
        assert rel_err(got[k], ref[k]) <= SUM_TOL, k


def test_backward_of_an_empty_sequence_passes_the_final_cotangent_through():
    h = ssd.SSD(2, 0, 2, 16, 16, 1, torch.float32)
    e = torch.empty(2, 0, 2, 16, device="cuda")
    A = -torch.ones(2, device="cuda")
    bc = torch.empty(2, 0, 1, 16, device="cuda")
    dfin = torch.randn(2, 2, 16, 16, device="cuda")
    g = h.backward(e, torch.empty(2, 0, 2, device="cuda"), A, bc, bc, e,
                   dfinal_states=dfin, initial_states=torch.randn(2, 2, 16, 16, device="cuda"))
    assert h.status() == 0
    assert torch.equal(g["dinitial_states"], dfin)
    assert torch.all(g["dA"] == 0) and torch.all(g["dD"] == 0)


def test_backward_bad_cu_seqlens_sets_status():
    w = I.random_small(4, "fp32", 1, 64, 2, 16, 16, 1, 64, varlen_tokens=64)
    inp = make(w, cu_seqlens=np.array([0, 40, 30, 64], dtype=np.int32))
    h = ssd.SSD(1, 64, 2, 16, 16, 1, torch.float32, max_docs=3)
    dy = torch.randn(1, 64, 2, 16, device="cuda")
    h.backward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], dy, inp["D"], inp["dt_bias"],
               cu_seqlens=inp["cu_seqlens"])
    assert h.status() == -6
    assert h.status() == 0
