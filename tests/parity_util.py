"""Shared helpers of the GPU parity tests (test infrastructure)."""

import numpy as np
import torch

import oracle
from structured_state_space_chunked_b200 import inputs as ssd_inputs
from structured_state_space_chunked_b200 import ssd

# max |y_gpu - y_ref| / max |y_ref| (and the same for final states)
TOL = {"fp32": 1e-4, "bf16": 2e-2}


def rel_err(got, ref, mask=None):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if mask is not None:
        got, ref = got[mask], ref[mask]
    denom = np.max(np.abs(ref)) if ref.size else 0.0
    if ref.size == 0:
        return 0.0
    return float(np.max(np.abs(got - ref)) / max(denom, 1e-30))


def to_np(t):
    return t.detach().to("cpu").double().numpy()


def gpu_run(w, inp, path=ssd.SSD_PATH_AUTO, chunk_size=None, handle=None, unit_columns=None):
    """Run the CUDA path through the C ABI; inputs already on the device."""
    max_docs = 0 if inp["cu_seqlens"] is None else inp["cu_seqlens"].numel() - 1
    bsz, L = inp["x"].shape[:2]
    h = handle or ssd.SSD(bsz, L, w.nheads, w.headdim, w.dstate, w.ngroups, w.torch_dtype,
                          max_docs=max_docs)
    if path != ssd.SSD_PATH_AUTO:
        h.force_path(path)
    if unit_columns is not None:
        h.tc_unit_columns(unit_columns)
    y, fin = h.forward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                       inp["dt_bias"], chunk_size or w.chunk_size, inp["initial_states"],
                       inp["cu_seqlens"])
    st = h.status()
    assert st == 0, f"device status {st}"
    torch.cuda.synchronize()
    return y, fin, h


def oracle_run(inp, heads=None):
    cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].cpu().numpy()
    return oracle.oracle_forward(inp["x"].cpu(), inp["dt"].cpu(), inp["A"].cpu(),
                                 inp["B"].cpu(), inp["C"].cpu(), inp["D"].cpu(),
                                 inp["dt_bias"].cpu(),
                                 None if inp["initial_states"] is None else inp["initial_states"].cpu(),
                                 cu_seqlens=cu, heads=heads)


def check(w, inp, y, fin, heads=None, tol=None):
    yr, fr = oracle_run(inp, heads)
    tol = tol or TOL[w.dtype]
    if heads is None:
        ey = rel_err(to_np(y), yr)
        ef = rel_err(to_np(fin), fr)
    else:
        ey = rel_err(to_np(y)[:, :, heads], yr[:, :, heads])
        ef = rel_err(to_np(fin)[:, heads], fr[:, heads])
    assert np.isfinite(ey) and np.isfinite(ef)
    assert ey <= tol, f"y rel err {ey:.3e} > {tol}"
    assert ef <= tol, f"final_states rel err {ef:.3e} > {tol}"
    return ey, ef


def make(w, device="cuda", **kw):
    return ssd_inputs.make_inputs(w, device=device, **kw)
