"""GPU parity where one persistent CTA walks several units (document, head, 64-column
slice) in a row, against the float64 oracle.

The tensor-core kernels give each CTA the units u, u + grid, ... of the problem, so a
CTA crosses unit boundaries whenever there are more units than SMs: the state restarts
from the unit's initial state, the previous unit's final state is written, and every
ring slot and barrier phase carries on across the boundary.  The workloads of the
benchmark with N = 256 have fewer units than SMs, so these cases make the crossing
happen on purpose: a batch of heads, and many packed documents of ragged lengths
(empty and one-token documents included), for the N = 256 kernel, and the N <= 128
shapes through the kernel that runs when a wait limit is set."""

import numpy as np
import pytest
import torch

from structured_state_space_chunked_b200 import inputs as I
from structured_state_space_chunked_b200 import ssd
from tests.parity_util import check, gpu_run, make

pytestmark = pytest.mark.gpu


def _lengths(seed, ndocs, hi):
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, hi, size=ndocs).tolist()
    lens[3] = 0     # empty documents
    lens[7] = 1     # one-token documents
    lens[11] = 0
    lens[12] = 256  # exactly two tiles
    lens[20] = 1
    return lens


def test_n256_batch_with_more_units_than_sms():
    # 4 x 32 heads x 2 slices = 256 units
    w = I.random_small(301, "bf16", 4, 300, 32, 128, 256, 2, 256, "normal0.1")
    inp = make(w)
    y, fin, h = gpu_run(w, inp)
    assert h.plan(256).path == ssd.SSD_PATH_TC
    check(w, inp, y, fin)


def test_n256_many_packed_documents():
    lens = _lengths(302, 60, 300)
    cu = I.cu_seqlens_from_lengths(lens)
    T = int(cu[-1])
    # 60 documents x 4 heads x 2 slices = 480 units
    w = I.random_small(302, "bf16", 1, T, 4, 128, 256, 1, 256, "normal0.1", varlen_tokens=T)
    inp = make(w, cu_seqlens=cu)
    y, fin, h = gpu_run(w, inp)
    assert h.plan(256).path == ssd.SSD_PATH_TC
    check(w, inp, y, fin)
    # an empty document hands its initial state straight through
    assert torch.equal(fin[3].cpu(), inp["initial_states"][3].cpu())


@pytest.mark.parametrize("N", [64, 128])
def test_wait_limited_kernel_many_packed_documents(N):
    lens = _lengths(303 + N, 60, 300)
    cu = I.cu_seqlens_from_lengths(lens)
    T = int(cu[-1])
    w = I.random_small(303 + N, "bf16", 1, T, 4, 64, N, 2, 256, "normal0.1", varlen_tokens=T)
    inp = make(w, cu_seqlens=cu)
    h = ssd.SSD(1, T, w.nheads, w.headdim, w.dstate, w.ngroups, w.torch_dtype, max_docs=len(lens))
    h.wait_limit_us(1000000)  # any limit but the default takes the kernel with bounded waits per role
    y, fin, _ = gpu_run(w, inp, handle=h)
    check(w, inp, y, fin)
