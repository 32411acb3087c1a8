"""GPU parity of ``ssd_step`` (one decode token per sequence, the recurrent mode of
"Transformers are SSMs", paperlayer.ai summary, §3.4.1) against the float64 step
oracle, and against the chunked forward: a prefill followed by steps equals one
forward over the longer sequence."""

import math

import numpy as np
import pytest
import torch

import oracle
from structured_state_space_chunked_b200 import inputs as I
from structured_state_space_chunked_b200 import ssd
from tests.parity_util import gpu_run, make, rel_err, to_np

pytestmark = pytest.mark.gpu


def _step_inputs(seed, dtype, b, H, P, N, G):
    r = np.random.default_rng(seed)
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    dev = "cuda"
    x = torch.tensor(r.standard_normal((b, H, P)), dtype=td, device=dev)
    dt = torch.tensor(r.standard_normal((b, H)), dtype=td, device=dev)
    A = torch.tensor(-np.exp(r.uniform(0, math.log(16), H)), dtype=torch.float32, device=dev)
    B = torch.tensor(r.standard_normal((b, G, N)) / math.sqrt(N), dtype=td, device=dev)
    C = torch.tensor(r.standard_normal((b, G, N)) / math.sqrt(N), dtype=td, device=dev)
    D = torch.tensor(r.standard_normal(H), dtype=torch.float32, device=dev)
    u = np.exp(r.uniform(math.log(1e-3), math.log(1e-1), H))
    bias = torch.tensor(np.log(np.expm1(u)), dtype=torch.float32, device=dev)
    state = torch.tensor(0.1 * r.standard_normal((b, H, N, P)), dtype=torch.float32, device=dev)
    return x, dt, A, B, C, D, bias, state


@pytest.mark.parametrize("case", [
    ("bf16", 5, 4, 64, 128, 2), ("fp32", 3, 2, 16, 16, 1), ("bf16", 2, 8, 128, 64, 4),
    ("bf16", 7, 6, 32, 256, 3), ("fp32", 1, 1, 4, 8, 1),
], ids=lambda c: "-".join(map(str, c)))
def test_step_matches_oracle(case):
    dtype, b, H, P, N, G = case
    x, dt, A, B, C, D, bias, state = _step_inputs(11 + b * H, dtype, b, H, P, N, G)
    s0 = state.clone()
    y = ssd.ssd_step(x, dt, A, B, C, state, D, bias)
    torch.cuda.synchronize()
    y_ref, s_ref = oracle.oracle_step(s0.cpu(), x.cpu(), dt.cpu(), A.cpu(), B.cpu(), C.cpu(),
                                      D.cpu(), bias.cpu())
    tol = 1e-4 if dtype == "fp32" else 2e-2
    assert rel_err(to_np(y), y_ref) <= tol
    assert rel_err(to_np(state), s_ref) <= tol


def test_step_without_optionals_and_fp32_output():
    x, dt, A, B, C, _, _, state = _step_inputs(3, "bf16", 4, 4, 64, 128, 1)
    s0 = state.clone()
    y = ssd.ssd_step(x, dt, A, B, C, state, out_dtype=torch.float32)
    assert y.dtype == torch.float32
    y_ref, s_ref = oracle.oracle_step(s0.cpu(), x.cpu(), dt.cpu(), A.cpu(), B.cpu(), C.cpu())
    assert rel_err(to_np(y), y_ref) <= 1e-4  # bf16 inputs, fp32 arithmetic and output
    assert rel_err(to_np(state), s_ref) <= 1e-4


@pytest.mark.parametrize("dtype,path", [("bf16", ssd.SSD_PATH_TC), ("fp32", ssd.SSD_PATH_SIMT)])
def test_prefill_then_steps_equal_one_longer_forward(dtype, path):
    # prefill L tokens with ssd_forward, then decode k tokens with ssd_step from its
    # final states: the outputs and final state equal one forward over L + k tokens
    b, L, k, H, P, N, G = 2, 256, 3, 4, 64, 128, 2
    if dtype == "fp32":
        P, N = 32, 16
    w = I.random_small(41, dtype, b, L + k, H, P, N, G, 128, "normal0.1")
    inp = make(w)
    y_full, f_full, _ = gpu_run(w, inp, path)
    pre = dict(inp)
    for key in ("x", "dt", "B", "C"):
        pre[key] = inp[key][:, :L].contiguous()
    wp = I.random_small(41, dtype, b, L, H, P, N, G, 128, "normal0.1")
    _, state, _ = gpu_run(wp, pre, path)
    tol = 1e-4 if dtype == "fp32" else 2e-2
    for t in range(L, L + k):
        y = ssd.ssd_step(inp["x"][:, t].contiguous(), inp["dt"][:, t].contiguous(), inp["A"],
                         inp["B"][:, t].contiguous(), inp["C"][:, t].contiguous(), state,
                         inp["D"], inp["dt_bias"])
        assert rel_err(to_np(y), to_np(y_full[:, t])) <= tol
    torch.cuda.synchronize()
    assert rel_err(to_np(state), to_np(f_full)) <= tol
