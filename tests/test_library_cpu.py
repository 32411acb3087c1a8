"""Host-side checks of libssd_b200 that need no GPU: the library loads, exports
every entry point include/ssd.h declares, validates descriptions, plans paths
and rejects bad calls before touching the device."""

import ctypes
import os
import re

import pytest
import torch

from structured_state_space_chunked_b200 import build as ssd_build
from structured_state_space_chunked_b200 import ssd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    ssd_build.build()
    return ssd.lib()


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"SSD_API\s+[\w\s\*]+?\b(ssd_\w+)\s*\(", txt))
    return names


def test_every_declared_symbol_is_exported(L):
    declared = _declared()
    assert declared, "no SSD_API declarations found"
    assert declared == set(ssd.ABI_SYMBOLS)
    for name in declared:
        assert hasattr(L, name), name


def test_version_and_error_strings(L):
    assert b"sm_100a" in L.ssd_version()
    for code, name in ssd.ERRORS.items():
        assert L.ssd_error_string(code).decode().startswith(name)
    assert L.ssd_error_string(-99) == b"SSD_ERR_UNKNOWN"


def _desc(**kw):
    base = dict(batch=2, seqlen=100, nheads=4, headdim=64, dstate=128, ngroups=2,
                dtype=torch.bfloat16, max_docs=0)
    base.update(kw)
    return ssd.make_desc(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(), 0),
    (dict(nheads=0), -1), (dict(headdim=-1), -1), (dict(batch=-1), -1),
    (dict(nheads=6, ngroups=4), -2), (dict(headdim=512), -2), (dict(dstate=300), -2),
    (dict(max_docs=4), -1),                  # packed documents need batch == 1
    (dict(batch=1, max_docs=4), 0),
    (dict(batch=0), 0), (dict(seqlen=0), 0),  # empty problems are valid
])
def test_validate_desc(L, kw, code):
    assert ssd.validate_desc(_desc(**kw)) == code


def test_bad_dtype_and_flags_rejected(L):
    d = _desc()
    d.in_dtype = 7
    assert ssd.validate_desc(d) == -1
    d = _desc()
    d.flags = 1
    assert ssd.validate_desc(d) == -1


@pytest.mark.parametrize("q", [0, 257, -3])
def test_plan_rejects_bad_chunk(L, q):
    with pytest.raises(ssd.SSDError) as e:
        ssd.plan(_desc(), q)
    assert e.value.code == -1


def test_plan_sizes_simt_workspace(L):
    d = _desc(dtype=torch.float32)
    p = ssd.plan(d, 64)
    assert p.path == ssd.SSD_PATH_SIMT
    nch = 2 * ((100 + 63) // 64)
    assert p.num_chunks_max == nch and p.num_docs == 2
    states = nch * 4 * 128 * 64 * 4
    assert p.workspace_bytes >= states + 2 * 4 * nch * 64 * 4
    # packed documents: one chunk slot of slack per document
    dv = _desc(batch=1, max_docs=8, dtype=torch.float32)
    pv = ssd.plan(dv, 64, num_docs=5)
    assert pv.num_chunks_max == (100 + 63) // 64 + 5
    with pytest.raises(ssd.SSDError):
        ssd.plan(dv, 64, num_docs=9)        # more documents than max_docs


def test_null_handle_and_missing_device_are_errors_not_crashes(L):
    vp = ctypes.c_void_p
    assert L.ssd_forward(None, None, None, None, None, None, None, None, 64, None, None, 0,
                         None, None, None) == -1
    assert L.ssd_get_status(None, None) == -1
    assert L.ssd_destroy(None) == 0
    assert L.ssd_set_option(None, 1, 0) == -1
    if not torch.cuda.is_available():
        h = vp()
        rc = L.ssd_create(ctypes.byref(_desc()), ctypes.byref(h))
        assert rc == -3 and not h.value


def test_step_validates_its_arguments_without_a_gpu():
    # ssd_step checks the descriptor before it touches the device
    L = ssd.lib()
    bad_len = ssd.make_desc(4, 2, 4, 64, 128, 1, torch.bfloat16)      # seqlen must be 1
    bad_p = ssd.make_desc(4, 1, 4, 6, 128, 1, torch.bfloat16)         # headdim % 4
    bad_g = ssd.make_desc(4, 1, 3, 64, 128, 2, torch.bfloat16)        # H % G
    empty = ssd.make_desc(0, 1, 4, 64, 128, 1, torch.bfloat16)        # no sequences: nothing to do
    null = [None] * 9
    assert L.ssd_step(ctypes.byref(bad_len), *null, None) == -1  # SSD_ERR_INVALID_ARG
    assert L.ssd_step(ctypes.byref(bad_p), *null, None) == -2  # SSD_ERR_UNSUPPORTED
    assert L.ssd_step(ctypes.byref(bad_g), *null, None) == -1  # SSD_ERR_INVALID_ARG
    assert L.ssd_step(ctypes.byref(empty), *null, None) == 0


def test_backward_refuses_a_missing_handle_without_a_gpu():
    # ssd_backward checks its handle before it touches the device
    L = ssd.lib()
    assert L.ssd_backward(None, *([None] * 9), 0, *([None] * 11)) == -1  # SSD_ERR_INVALID_ARG


def test_feature_map_dims_without_a_gpu():
    assert [ssd.feature_map_dim(k, 8) for k in range(5)] == [8, 8, 8, 73, 64]
    assert ssd.lib().ssd_feature_map_dim(7, 8) == -1
    assert ssd.lib().ssd_forward_ext(None, *([None] * 7), 64, None, 0, 1, 0, None, None, None) == -1


def test_context_parallel_entries_validate_their_arguments_without_a_gpu():
    # every check below returns before the device is touched
    L = ssd.lib()
    d = ssd.make_desc(2, 128, 4, 64, 128, 1, torch.bfloat16)
    packed = ssd.make_desc(1, 128, 4, 64, 128, 1, torch.bfloat16, max_docs=3)  # batch mode only
    bad_g = ssd.make_desc(2, 128, 3, 64, 128, 2, torch.bfloat16)
    empty = ssd.make_desc(0, 128, 4, 64, 128, 1, torch.bfloat16)
    assert L.ssd_cp_logdecay(None, None, None, None, None, None, None) == -1
    assert L.ssd_cp_logdecay(ctypes.byref(packed), None, None, None, None, None, None) == -1
    assert L.ssd_cp_logdecay(ctypes.byref(bad_g), None, None, None, None, None, None) == -1
    assert L.ssd_cp_logdecay(ctypes.byref(d), None, None, None, None, None, None) == -1   # null arrays
    assert L.ssd_cp_logdecay(ctypes.byref(empty), None, None, None, None, None, None) == 0
    for rank, nranks in ((2, 2), (-1, 2), (0, 0)):
        assert L.ssd_cp_combine(ctypes.byref(d), rank, nranks, None, None, None, None, None, None) == -1
    assert L.ssd_cp_combine(ctypes.byref(d), 0, 2, None, None, None, None, None, None) == -1
    assert L.ssd_cp_correct(ctypes.byref(d), None, None, None, None, None, None) == -1


def test_forward_ext_refuses_a_missing_handle_and_feature_map_dim_checks_without_a_gpu():
    # (the option checks behind a valid handle are GPU tests in test_ext_gpu.py)
    L = ssd.lib()
    assert L.ssd_forward_ext(None, *([None] * 7), 64, None, 0, 1, 0, None, None, None) == -1
    assert L.ssd_feature_map_dim(9, 16) == -1          # unknown feature map
    assert L.ssd_feature_map_dim(ssd.SSD_FMAP_BASED, 0) == -1
    assert L.ssd_feature_map_dim(ssd.SSD_FMAP_BASED, 8) == 1 + 8 + 64
    assert L.ssd_feature_map_dim(ssd.SSD_FMAP_REBASED, 8) == 64
