"""GPU parity of ssd_forward_ext (feature maps on B and C, denominator normalisation)
against the float64 oracle ("Transformers are SSMs", paperlayer.ai summary, §7.3 and
App. D.4).  Tolerances as for the plain forward (1e-4 fp32, 2e-2 bf16, relative to
max |ref|).  With normalisation the output is num / den + D x.  Rounding errors
e_n <= tol max|num| of the numerator and e_d <= tol max|den| of the denominator
give |y_gpu - y_ref| den <= tol (max|num| + |num / den| max|den|) to first order,
so that is the per-token bound of the normalised cases (a wrong divisor breaks it
by a wide margin); tokens whose reference denominator is under 1 % of the median
are left out (ReLU and ReBased maps can make it near zero)."""

import numpy as np
import pytest
import torch

import oracle
from structured_state_space_chunked_b200 import inputs as I
from structured_state_space_chunked_b200 import ssd
from tests.parity_util import TOL, make, rel_err, to_np

pytestmark = pytest.mark.gpu

CASES = [
    # dtype, batch, seqlen, H, P, N, G, feature map, normalize, varlen tokens, chunk
    # chunk 64: the numerator runs on the CUDA-core path (the tensor-core kernel
    # needs chunks of a multiple of 128 tokens)
    ("bf16", 2, 300, 4, 64, 128, 1, ssd.SSD_FMAP_SILU, False, 0, 64),
    ("bf16", 2, 300, 4, 64, 64, 2, ssd.SSD_FMAP_RELU, True, 0, 64),
    ("fp32", 1, 200, 3, 16, 8, 1, ssd.SSD_FMAP_BASED, True, 0, 64),
    ("bf16", 1, 257, 2, 64, 8, 1, ssd.SSD_FMAP_REBASED, True, 0, 64),
    ("bf16", 1, 0, 2, 64, 16, 1, ssd.SSD_FMAP_BASED, True, 1000, 64),
    ("fp32", 2, 100, 2, 32, 16, 1, ssd.SSD_FMAP_NONE, True, 0, 64),
    ("fp32", 2, 130, 2, 32, 16, 2, ssd.SSD_FMAP_RELU, False, 0, 64),
    # chunk 256, bf16, mapped dstate a multiple of 16: the numerator runs on the
    # tensor cores over the mapped B and C (the configuration the benchmark times)
    ("bf16", 2, 600, 4, 64, 64, 1, ssd.SSD_FMAP_SILU, False, 0, 256),
    ("bf16", 2, 520, 4, 64, 128, 2, ssd.SSD_FMAP_RELU, True, 0, 256),
    ("bf16", 1, 700, 2, 64, 8, 1, ssd.SSD_FMAP_REBASED, True, 0, 256),
    ("bf16", 1, 0, 4, 64, 8, 1, ssd.SSD_FMAP_REBASED, True, 1500, 256),
    # the denominator's block form with full head blocks (24 heads of one group, as in
    # the 130M layer), a ragged head block (12 heads per group: 8 + 4) over packed
    # documents, and the largest mapped dstate it takes (256, fp32)
    ("bf16", 2, 700, 24, 64, 128, 1, ssd.SSD_FMAP_RELU, True, 0, 256),
    ("bf16", 1, 0, 24, 64, 64, 2, ssd.SSD_FMAP_RELU, True, 1300, 256),
    ("fp32", 1, 300, 3, 16, 16, 1, ssd.SSD_FMAP_REBASED, True, 0, 64),
    # bf16 with a mapped dstate that is no multiple of 8 (Based, N = 8 -> 73): the
    # denominator's element-by-element staging and its products over zero-padded columns
    ("bf16", 2, 300, 8, 64, 8, 1, ssd.SSD_FMAP_BASED, True, 0, 64),
    # 128 or more tensor-core units (more than 3/4 of a B200's 148 SMs): the denominator
    # first, the division folded into the numerator kernel's output epilogue
    ("bf16", 2, 700, 64, 64, 128, 1, ssd.SSD_FMAP_RELU, True, 0, 256),
    ("bf16", 1, 0, 64, 64, 64, 2, ssd.SSD_FMAP_RELU, True, 1500, 256),
]
IDS = ["silu-simt", "relu-norm-simt", "based-norm-simt-fp32", "rebased-norm-simt",
       "based-norm-packed-simt", "none-norm-fp32", "relu-fp32",
       "silu-tc", "relu-norm-tc", "rebased-norm-tc", "rebased-norm-packed-tc",
       "relu-norm-tc-h24", "relu-norm-packed-tc-hpg12", "rebased-norm-fp32-n256",
       "based-norm-bf16-n73", "relu-norm-tc-folded", "relu-norm-packed-tc-folded"]


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_forward_ext_matches_oracle(case):
    dtype, b, L, H, P, N, G, fmap, norm, vt, Q = case
    w = I.random_small(900 + N + P, dtype, b, L, H, P, N, G, Q, "zero", vt)
    inp = make(w)
    bsz, Lr = inp["x"].shape[:2]
    max_docs = 0 if inp["cu_seqlens"] is None else inp["cu_seqlens"].numel() - 1
    h = ssd.SSD(bsz, Lr, H, P, N, G, w.torch_dtype, max_docs=max_docs)
    if Q == 256:
        # the numerator takes the plain forward's path at the mapped dstate: the
        # tensor-core kernel here
        n2 = ssd.feature_map_dim(fmap, N)
        mapped = ssd.make_desc(bsz, Lr, H, P, n2, G, w.torch_dtype, max_docs=max_docs)
        assert ssd.plan(mapped, Q, max_docs).path == ssd.SSD_PATH_TC
    y, fin = h.forward_ext(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                           inp["dt_bias"], Q, feature_map=fmap, normalize=norm,
                           cu_seqlens=inp["cu_seqlens"])
    assert h.status() == 0
    torch.cuda.synchronize()
    check_against_oracle(dtype, inp, y, fin, fmap, norm, N)


def check_against_oracle(dtype, inp, y, fin, fmap, norm, N):
    cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].cpu().numpy()
    cpu = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
    yr, fr = oracle.oracle_forward_ext(cpu["x"], cpu["dt"], cpu["A"], cpu["B"], cpu["C"], cpu["D"],
                                       cpu["dt_bias"], fmap, norm, cu_seqlens=cu)
    yg = to_np(y)
    mask = np.ones(yr.shape, dtype=bool)
    if norm:
        Bf = oracle.oracle_feature_map(cpu["B"], fmap)
        Cf = oracle.oracle_feature_map(cpu["C"], fmap)
        den, _ = oracle.oracle_forward(np.ones(yr.shape[:-1] + (1,)), cpu["dt"], cpu["A"], Bf, Cf,
                                       None, cpu["dt_bias"], cu_seqlens=cu)
        ok = np.abs(den[..., 0]) > 0.01 * np.median(np.abs(den))
        assert ok.mean() > 0.8
        mask = np.broadcast_to(ok[..., None], yr.shape)
    tol = TOL[dtype]
    if norm:
        dd = np.broadcast_to(den, yr.shape)
        D64 = cpu["D"].double().numpy()
        ratio = yr - D64[None, None, :, None] * cpu["x"].double().numpy()  # num / den
        scale = np.max(np.abs((ratio * dd)[mask])) + np.abs(ratio) * np.max(np.abs(dd[mask]))
        e = float(np.max((np.abs(yg - yr) * dd / scale)[mask]))
    else:
        e = rel_err(yg, yr, mask)
    assert e <= tol, f"y rel err {e:.3e}"
    assert fin.shape[2] == ssd.feature_map_dim(fmap, N)
    ef = rel_err(to_np(fin), fr)
    assert ef <= tol, f"final_states rel err {ef:.3e}"



def test_forward_ext_repeated_calls_on_one_handle():
    """Three normalised calls on one handle (the denominator runs on the handle's second
    stream), each checked against the oracle, with different inputs and a packed one."""
    L, H, P, N, G = 1400, 24, 64, 128, 1
    outs = []
    h = None
    for seed, vt in ((31, 0), (32, 0), (33, L)):
        w = I.random_small(seed, "bf16", 1, 0 if vt else L, H, P, N, G, 256, "zero", vt)
        inp = make(w)
        assert inp["x"].shape[:2] == (1, L)
        if h is None:
            h = ssd.SSD(1, L, H, P, N, G, torch.bfloat16, max_docs=L)
        y, fin = h.forward_ext(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                               inp["dt_bias"], 256, feature_map=ssd.SSD_FMAP_RELU, normalize=True,
                               cu_seqlens=inp["cu_seqlens"])
        outs.append((inp, y.clone(), fin.clone()))
    torch.cuda.synchronize()
    assert h.status() == 0
    for inp, y, fin in outs:
        check_against_oracle("bf16", inp, y, fin, ssd.SSD_FMAP_RELU, True, N)


def test_unknown_feature_map_is_refused():
    w = I.random_small(1, "bf16", 1, 64, 2, 64, 64, 1, 64)
    inp = make(w)
    h = ssd.SSD(1, 64, 2, 64, 64, 1, torch.bfloat16)
    with pytest.raises(ssd.SSDError):
        h.forward_ext(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], feature_map=9)


def test_normalize_outside_zero_one_is_refused():
    w = I.random_small(2, "bf16", 1, 64, 2, 64, 64, 1, 64)
    inp = make(w)
    h = ssd.SSD(1, 64, 2, 64, 64, 1, torch.bfloat16)
    y = torch.empty_like(inp["x"])
    rc = ssd.lib().ssd_forward_ext(h._h, *(ssd._ptr(inp[k]) for k in ("x", "dt", "A", "B", "C")),
                                   None, None, 64, None, 0, ssd.SSD_FMAP_RELU, 2, ssd._ptr(y),
                                   None, None)
    assert rc == -1


def test_forward_ext_bad_cu_seqlens_sets_status():
    w = I.random_small(4, "bf16", 1, 0, 2, 64, 64, 1, 64, "zero", 256)
    inp = make(w, cu_seqlens=np.array([0, 200, 100, 256], dtype=np.int32))
    h = ssd.SSD(1, 256, 2, 64, 64, 1, torch.bfloat16, max_docs=3)
    h.forward_ext(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], inp["dt_bias"], 64,
                  feature_map=ssd.SSD_FMAP_RELU, normalize=True, cu_seqlens=inp["cu_seqlens"])
    assert h.status() == -6
