"""GPU parity: the CUDA path, called through the C ABI, against the float64
oracle on the same seeded inputs.  Pass rule (max |err| / max |y_ref|, the same
for final states): 1e-4 for fp32 inputs, 2e-2 for bf16 inputs with fp32
accumulation."""

import numpy as np
import pytest
import torch

from structured_state_space_chunked_b200 import inputs as I
from structured_state_space_chunked_b200 import ssd
from tests.parity_util import TOL, check, gpu_run, make, oracle_run, rel_err, to_np

pytestmark = pytest.mark.gpu

PATHS = [ssd.SSD_PATH_SIMT, ssd.SSD_PATH_TC]


def _tc_ok(w, chunk):
    d = ssd.make_desc(w.batch if not w.varlen_tokens else 1,
                      w.seqlen if not w.varlen_tokens else w.varlen_tokens,
                      w.nheads, w.headdim, w.dstate, w.ngroups, w.torch_dtype,
                      max_docs=1 if w.varlen_tokens else 0)
    return ssd.plan(d, chunk, 1 if w.varlen_tokens else 0).path == ssd.SSD_PATH_TC


SMALL = [
    # dtype, batch, seqlen, H, P, N, G, Q, init
    ("fp32", 1, 256, 2, 16, 16, 1, 64, "zero"),
    ("fp32", 2, 300, 4, 32, 24, 2, 100, "normal0.1"),
    ("bf16", 2, 300, 4, 64, 128, 1, 128, "zero"),
    ("bf16", 1, 515, 6, 64, 128, 3, 256, "normal0.1"),
    ("bf16", 2, 384, 4, 128, 64, 2, 256, "zero"),
    ("bf16", 1, 333, 4, 128, 128, 4, 128, "normal0.1"),
    ("bf16", 1, 290, 2, 128, 256, 1, 256, "normal0.1"),
    ("bf16", 3, 129, 2, 64, 128, 2, 128, "normal0.1"),
    ("bf16", 1, 200, 2, 256, 128, 1, 128, "normal0.1"),
    ("bf16", 2, 250, 4, 64, 64, 2, 256, "normal0.1"),
    ("bf16", 1, 140, 2, 64, 32, 1, 128, "zero"),
]


@pytest.mark.parametrize("path", PATHS, ids=["simt", "tc"])
@pytest.mark.parametrize("case", SMALL, ids=lambda c: "-".join(map(str, c)))
def test_small_shapes(case, path):
    dtype, b, L, H, P, N, G, Q, init = case
    w = I.random_small(7 + L, dtype, b, L, H, P, N, G, Q, init)
    if path == ssd.SSD_PATH_TC and not _tc_ok(w, Q):
        pytest.skip("shape outside the tensor-core path")
    inp = make(w)
    y, fin, _ = gpu_run(w, inp, path)
    check(w, inp, y, fin)


def _wide_ok(w):
    # 128-column units: N <= 128 and whole units in one B/C group
    if w.dtype != "bf16" or w.dstate > 128 or w.chunk_size % 128:
        return False
    if w.headdim % 128 == 0:
        return w.headdim <= 256
    return w.headdim == 64 and (w.nheads // w.ngroups) % 2 == 0


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "-".join(map(str, c)))
def test_small_shapes_128_column_units(case):
    dtype, b, L, H, P, N, G, Q, init = case
    w = I.random_small(7 + L, dtype, b, L, H, P, N, G, Q, init)
    if not _wide_ok(w):
        pytest.skip("shape outside 128-column units")
    inp = make(w)
    y, fin, _ = gpu_run(w, inp, ssd.SSD_PATH_TC, unit_columns=128)
    check(w, inp, y, fin)


@pytest.mark.parametrize("name", ["mamba2_130m_layer_b4_L2048", "varlen_32k_H32_P64_N128",
                                  "long_L2048_H64_P128_N128_G8"])
def test_workloads_128_column_units_sampled(name):
    w = I.workload(name)
    inp = make(w)
    y, fin, _ = gpu_run(w, inp, ssd.SSD_PATH_TC, unit_columns=128)
    check(w, inp, y, fin, heads=[0, 1, w.nheads - 1])


def test_128_column_units_unsupported_shape_is_refused():
    w = I.random_small(3, "bf16", 1, 256, 3, 64, 128, 3, 128, "zero")  # H/G = 1: no head pair
    inp = make(w)
    with pytest.raises(ssd.SSDError):
        gpu_run(w, inp, ssd.SSD_PATH_TC, unit_columns=128)


@pytest.mark.parametrize("Q", [1, 3, 16, 64, 100, 128, 256])
def test_every_chunk_size_gives_the_same_answer(Q):
    w = I.random_small(3, "fp32", 2, 257, 3, 32, 16, 1, Q, "normal0.1")
    inp = make(w)
    y, fin, _ = gpu_run(w, inp, ssd.SSD_PATH_SIMT, chunk_size=Q)
    check(w, inp, y, fin)


def test_tiny_fp32_workload():
    w = I.workloads()[0]
    inp = make(w)
    y, fin, _ = gpu_run(w, inp)
    check(w, inp, y, fin)


def test_mamba2_130m_layer_full_oracle():
    w = I.workload("mamba2_130m_layer_b4_L2048")
    inp = make(w)
    y, fin, _ = gpu_run(w, inp)
    check(w, inp, y, fin)


def test_mamba2_2p7b_layer_all_heads():
    w = I.workload("mamba2_2p7b_layer_b8_L4096")
    inp = make(w)
    y, fin, _ = gpu_run(w, inp)
    check(w, inp, y, fin)


LONG = [w for w in I.workloads() if w.name.startswith("long_")]


@pytest.mark.parametrize("w", [w for w in LONG if w.seqlen <= 16384], ids=lambda w: w.name)
def test_long_sequence_all_heads(w):
    inp = make(w)
    y, fin, h = gpu_run(w, inp)
    check(w, inp, y, fin)
    del y, fin, inp, h
    torch.cuda.empty_cache()


@pytest.mark.parametrize("w", [w for w in LONG if w.seqlen > 16384], ids=lambda w: w.name)
def test_long_sequence_65536_sampled_heads(w):
    # host memory bounds the float64 reference here: heads from both halves of the
    # head range and of two different B/C groups, every token and state element
    inp = make(w)
    y, fin, h = gpu_run(w, inp)
    check(w, inp, y, fin, heads=[0, 5, 33, 60, 63])
    del y, fin, inp, h
    torch.cuda.empty_cache()


def test_varlen_packed_documents_all_heads():
    w = I.workload("varlen_32k_H32_P64_N128")
    inp = make(w)
    y, fin, _ = gpu_run(w, inp)
    check(w, inp, y, fin)


@pytest.mark.parametrize("path", PATHS, ids=["simt", "tc"])
def test_varlen_edge_documents(path):
    # empty documents, single-token documents, one longer than several chunks
    lens = [1, 0, 300, 17, 0, 1, 129, 128, 2]
    cu = I.cu_seqlens_from_lengths(lens)
    T = int(cu[-1])
    w = I.random_small(21, "bf16", 1, T, 4, 64, 128, 1, 128, "normal0.1", varlen_tokens=T)
    if path == ssd.SSD_PATH_TC and not _tc_ok(w, 128):
        pytest.skip("shape outside the tensor-core path")
    inp = make(w, cu_seqlens=cu)
    y, fin, _ = gpu_run(w, inp, path)
    check(w, inp, y, fin)
    # an empty document hands its initial state straight through
    assert torch.equal(fin[1].cpu(), inp["initial_states"][1].cpu())


def test_packed_equals_separate_calls():
    lens = [70, 5, 181]
    cu = I.cu_seqlens_from_lengths(lens)
    T = int(cu[-1])
    w = I.random_small(5, "fp32", 1, T, 2, 32, 16, 1, 64, "normal0.1", varlen_tokens=T)
    inp = make(w, cu_seqlens=cu)
    y, fin, _ = gpu_run(w, inp, ssd.SSD_PATH_SIMT)
    for d in range(len(lens)):
        s, e = int(cu[d]), int(cu[d + 1])
        sub = dict(inp)
        for k in ("x", "dt", "B", "C"):
            sub[k] = inp[k][:, s:e].contiguous()
        sub["initial_states"] = inp["initial_states"][d:d + 1].contiguous()
        sub["cu_seqlens"] = None
        ws = I.random_small(5, "fp32", 1, e - s, 2, 32, 16, 1, 64)
        ys, fs, _ = gpu_run(ws, sub, ssd.SSD_PATH_SIMT)
        assert rel_err(to_np(y[:, s:e]), to_np(ys)) < 1e-6
        assert rel_err(to_np(fin[d]), to_np(fs[0])) < 1e-6


def test_state_handoff_across_calls():
    # two calls chained through final_states -> initial_states equal one call
    w = I.random_small(9, "bf16", 2, 512, 4, 64, 128, 1, 256, "normal0.1")
    inp = make(w)
    y, fin, _ = gpu_run(w, inp)
    t0 = 256
    a = {k: (v[:, :t0].contiguous() if k in ("x", "dt", "B", "C") else v) for k, v in inp.items()}
    b = {k: (v[:, t0:].contiguous() if k in ("x", "dt", "B", "C") else v) for k, v in inp.items()}
    wa = I.random_small(9, "bf16", 2, t0, 4, 64, 128, 1, 256)
    ya, fa, _ = gpu_run(wa, a)
    b["initial_states"] = fa
    yb, fb, _ = gpu_run(wa, b)
    tol = TOL["bf16"]
    assert rel_err(to_np(torch.cat([ya, yb], 1)), to_np(y)) < tol
    assert rel_err(to_np(fb), to_np(fin)) < tol


def test_bad_cu_seqlens_sets_status_and_writes_nothing():
    w = I.random_small(4, "fp32", 1, 64, 2, 16, 16, 1, 32, varlen_tokens=64)
    inp = make(w, cu_seqlens=np.array([0, 40, 30, 64], dtype=np.int32))
    h = ssd.SSD(1, 64, 2, 16, 16, 1, torch.float32, max_docs=3)
    y = torch.full((1, 64, 2, 16), 7.0, device="cuda")
    h.forward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], inp["dt_bias"], 32,
              None, inp["cu_seqlens"], y=y, return_final_states=False)
    assert h.status() == -6
    assert torch.all(y == 7.0)
    assert h.status() == 0  # cleared by the read


def test_empty_sequence_and_null_optionals():
    h = ssd.SSD(2, 0, 2, 16, 16, 1, torch.float32)
    A = -torch.ones(2, device="cuda")
    e = torch.empty(2, 0, 2, 16, device="cuda")
    init = torch.randn(2, 2, 16, 16, device="cuda")
    y, fin = h.forward(e, torch.empty(2, 0, 2, device="cuda"), A,
                       torch.empty(2, 0, 1, 16, device="cuda"), torch.empty(2, 0, 1, 16, device="cuda"),
                       None, None, 64, init)
    assert h.status() == 0
    assert torch.equal(fin, init)


@pytest.mark.parametrize("case", [
    # dtype, batch, seqlen, H, P, N, G, Q, varlen lengths (None: batch mode), pinned
    ("bf16", 9, 200, 4, 64, 128, 1, 256, None, True),
    ("bf16", 1, 0, 4, 64, 128, 1, 128, [1, 0, 300, 17, 0, 1, 129, 128, 2, 40, 260], False),
    ("bf16", 1, 0, 4, 64, 128, 1, 128, [700], True),
    ("fp32", 3, 150, 2, 32, 16, 1, 64, None, False),
], ids=["batch9-pinned", "varlen11", "one-doc", "fp32-batch3"])
def test_host_entry_point_pipelined_equals_device_call(case):
    # ssd_forward_host splits the documents into groups whose copies and compute
    # overlap; every group computes the same units as one device call
    dtype, b, L, H, P, N, G, Q, lens, pinned = case
    cu = None
    if lens is not None:
        cu = I.cu_seqlens_from_lengths(lens)
        L = int(cu[-1])
    w = I.random_small(31 + L, dtype, b, L, H, P, N, G, Q, "normal0.1",
                       varlen_tokens=L if lens is not None else 0)
    inp = make(w, cu_seqlens=cu)
    y1, f1, h = gpu_run(w, inp)
    host = {k: (None if v is None else (v.cpu().pin_memory() if pinned else v.cpu()))
            for k, v in inp.items()}
    yh, fh = h.forward_host(host["x"], host["dt"], host["A"], host["B"], host["C"], host["D"],
                            host["dt_bias"], Q, host["initial_states"], host["cu_seqlens"])
    assert h.status() == 0
    assert torch.equal(yh, y1.cpu()) and torch.equal(fh, f1.cpu())


def test_deterministic_and_host_entry_point_agree():
    w = I.random_small(12, "bf16", 2, 300, 4, 64, 128, 1, 256, "normal0.1")
    inp = make(w)
    y1, f1, h = gpu_run(w, inp)
    y2, f2, _ = gpu_run(w, inp, handle=h)
    assert torch.equal(y1, y2) and torch.equal(f1, f2)
    host = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
    yh, fh = h.forward_host(host["x"], host["dt"], host["A"], host["B"], host["C"], host["D"],
                            host["dt_bias"], 256, host["initial_states"])
    assert torch.equal(yh, y1.cpu()) and torch.equal(fh, f1.cpu())
