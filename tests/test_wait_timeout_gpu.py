"""Failure detection without a GPU fault: a device-side wait that runs out.

The tensor-core forward bounds every mbarrier wait.  With the failure-path
option SSD_OPT_TEST_FORCE_TIMEOUT the kernel's first epilogue wait is on a
barrier that nothing completes; after the SSD_OPT_WAIT_LIMIT_US bound it gives
up, records SSD_ERR_TIMEOUT in the handle's status word, and every role of the
kernel unwinds (the MMA issuer waits for its issued products and the TMA
producer for its loads before tensor memory is freed).  The test reads the
status on the host, then runs a normal call on the same handle and checks it
against the float64 oracle: the context and the handle stayed usable."""

import pytest
import torch

from structured_state_space_chunked_b200 import inputs as I
from structured_state_space_chunked_b200 import ssd
from tests.parity_util import check, make

pytestmark = pytest.mark.gpu

SSD_ERR_TIMEOUT = -4


@pytest.mark.parametrize("case", [
    # batch, seqlen, H, P, N, G, Q
    (2, 640, 4, 64, 128, 1, 256),
    (1, 300, 2, 128, 64, 2, 128),
    (2, 700, 4, 128, 256, 2, 256),
], ids=["b2-L640-N128", "b1-L300-P128-N64", "b2-L700-P128-N256"])
def test_forced_wait_runs_out_then_the_handle_computes_again(case):
    b, L, H, P, N, G, Q = case
    w = I.random_small(70 + L, "bf16", b, L, H, P, N, G, Q, "normal0.1")
    inp = make(w)
    h = ssd.SSD(b, L, H, P, N, G, torch.bfloat16)
    assert h.plan(Q).path == ssd.SSD_PATH_TC
    args = (inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], inp["dt_bias"], Q,
            inp["initial_states"])
    h.wait_limit_us(20000)  # 20 ms
    h.force_timeout(True)
    h.forward(*args)
    assert h.status() == SSD_ERR_TIMEOUT
    assert h.status() == 0  # cleared by the read
    # a second forced timeout on the same handle, then a normal call
    h.forward(*args)
    assert h.status() == SSD_ERR_TIMEOUT
    h.force_timeout(False)
    h.wait_limit_us(2000000)
    y, fin = h.forward(*args)
    assert h.status() == 0
    torch.cuda.synchronize()
    check(w, inp, y, fin)


def test_wait_limit_option_range():
    h = ssd.SSD(1, 128, 2, 64, 64, 1, torch.bfloat16)
    for bad in (0, -5, 60000001):
        with pytest.raises(ssd.SSDError):
            h.wait_limit_us(bad)
    assert ssd.lib().ssd_set_option(h._h, ssd.SSD_OPT_TEST_FORCE_TIMEOUT, 2) == -1
