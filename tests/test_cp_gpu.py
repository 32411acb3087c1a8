"""GPU parity of the context-parallel device steps (ssd_cp_logdecay, ssd_cp_combine,
ssd_cp_correct): a sequence cut into rank slices, each slice run by ssd_forward from
a zero state and then corrected with the state entering it, equals one forward over
the whole sequence and the float64 oracle ("Transformers are SSMs", paperlayer.ai
summary, §8.2 and §6.2).  The ranks are emulated one after another in this process;
the all-gather between them is a stack (the collective itself is tested on CPU)."""

import pytest
import torch

from structured_state_space_chunked_b200 import dist as sdist
from structured_state_space_chunked_b200 import inputs as I
from structured_state_space_chunked_b200 import ssd
from tests.parity_util import TOL, check, gpu_run, make, oracle_run, rel_err, to_np

pytestmark = pytest.mark.gpu


def _cp_run(w, inp, cuts, path):
    ys, S, ld, cs, parts = [], [], [], [], []
    for t0, t1 in zip(cuts[:-1], cuts[1:]):
        part = {k: inp[k][:, t0:t1].contiguous() for k in ("x", "dt", "B", "C")}
        h = ssd.SSD(w.batch, t1 - t0, w.nheads, w.headdim, w.dstate, w.ngroups, w.torch_dtype)
        h.force_path(path)
        y, s = h.forward(part["x"], part["dt"], inp["A"], part["B"], part["C"], inp["D"],
                         inp["dt_bias"], w.chunk_size, None, None)
        c, l = ssd.cp_logdecay(part["dt"], inp["A"], inp["dt_bias"], headdim=w.headdim,
                               dstate=w.dstate, ngroups=w.ngroups)
        ys.append(y), S.append(s), ld.append(l), cs.append(c), parts.append(part)
    S_all, ld_all = torch.stack(S), torch.stack(ld)
    finals = []
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for r in range(len(ys)):
        h_in, fin = ssd.cp_combine(r, S_all, ld_all, inp["initial_states"], dt_dtype=w.torch_dtype)
        ssd.cp_correct(parts[r]["C"], cs[r], h_in, ys[r], status=status)
        finals.append(fin)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return torch.cat(ys, dim=1), finals[-1]


@pytest.mark.parametrize("case", [
    # dtype, batch, seqlen, H, P, N, G, Q, init, cuts
    ("bf16", 2, 600, 4, 64, 128, 2, 256, "normal0.1", [0, 128, 384, 600]),
    ("bf16", 1, 1024, 2, 128, 64, 1, 128, "zero", [0, 512, 1024]),
    ("fp32", 2, 300, 3, 32, 16, 1, 64, "normal0.1", [0, 77, 150, 151, 300]),
    ("bf16", 2, 700, 2, 256, 128, 1, 128, "normal0.1", [0, 300, 700]),
    ("bf16", 1, 520, 4, 64, 256, 2, 128, "normal0.1", [0, 130, 260, 520]),
    ("fp32", 3, 256, 2, 64, 64, 1, 64, "normal0.1", [0, 100, 256]),
], ids=["bf16-3ranks", "bf16-2ranks", "fp32-4ranks", "bf16-P256", "bf16-N256", "fp32-P64N64"])
def test_context_parallel_slices_equal_one_forward(case):
    dtype, b, L, H, P, N, G, Q, init, cuts = case
    w = I.random_small(61 + L, dtype, b, L, H, P, N, G, Q, init)
    inp = make(w)
    path = ssd.SSD_PATH_TC if dtype == "bf16" else ssd.SSD_PATH_SIMT
    y_cp, fin_cp = _cp_run(w, inp, cuts, path)
    check(w, inp, y_cp, fin_cp)                       # against the float64 oracle
    y_full, f_full, _ = gpu_run(w, inp, path)         # and against one device forward
    tol = TOL[dtype]
    assert rel_err(to_np(y_cp), to_np(y_full)) <= tol
    assert rel_err(to_np(fin_cp), to_np(f_full)) <= tol


def test_context_parallel_forward_on_one_rank_is_the_plain_forward():
    w = I.random_small(5, "bf16", 2, 384, 4, 64, 128, 1, 256, "normal0.1")
    inp = make(w)
    h = ssd.SSD(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups, w.torch_dtype)
    y, fin = sdist.context_parallel_forward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"],
                                            inp["D"], inp["dt_bias"], w.chunk_size,
                                            inp["initial_states"], group=None, handle=h)
    torch.cuda.synchronize()
    check(w, inp, y, fin)


@pytest.mark.parametrize("P,N,G,L,out,tc", [
    (64, 128, 2, 333, torch.float32, True), (128, 64, 1, 333, torch.bfloat16, True),
    (256, 256, 1, 333, torch.float32, True), (192, 128, 2, 1000, torch.bfloat16, True),
    (64, 16, 1, 333, torch.float32, False), (64, 128, 1, 100, torch.bfloat16, False)],
    ids=["P64N128-f32", "P128N64-bf16", "P256N256-f32", "P192N128-bf16", "P64N16-cudacores",
         "L100-cudacores"])
def test_correction_equals_its_definition(P, N, G, L, out, tc):
    """y + exp(cs) C H_in for random operands, against the same sum in float64 with H_in
    rounded to bf16 where the tensor cores take it as a bf16 operand (the CUDA-core
    fallback keeps it in fp32)."""
    g = torch.Generator().manual_seed(P * 1000 + N + L)
    b, H = 2, 4
    C = torch.randn(b, L, G, N, generator=g).to(torch.bfloat16)
    cs = -torch.rand(b, L, H, generator=g).cumsum(1) * 0.05
    h_in = torch.randn(b, H, N, P, generator=g)
    y = torch.randn(b, L, H, P, generator=g).to(out)
    Cg = C.double().repeat_interleave(H // G, dim=2)                    # [b, L, H, N]
    hb = (h_in.to(torch.bfloat16) if tc else h_in).double()
    ref = y.double() + cs.double().exp()[..., None] * torch.einsum("blhn,bhnp->blhp", Cg, hb)
    yd = y.cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ssd.cp_correct(C.cuda(), cs.cuda(), h_in.cuda(), yd, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    err = (yd.double().cpu() - ref).abs().max() / ref.abs().max()
    assert err <= (2e-2 if out == torch.bfloat16 else 1e-4)


@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_correction_with_several_items_per_cta(out):
    """Enough (batch, head, tile run) items that each persistent CTA of the tensor-core
    correction takes several in a row (its C-tile prefetch and barrier phases carry
    across items), against the definition in float64."""
    g = torch.Generator().manual_seed(777)
    b, L, H, P, N, G = 4, 2048, 48, 64, 128, 1
    C = torch.randn(b, L, G, N, generator=g).to(torch.bfloat16)
    cs = -torch.rand(b, L, H, generator=g).cumsum(1) * 0.002
    h_in = torch.randn(b, H, N, P, generator=g)
    y = torch.randn(b, L, H, P, generator=g).to(out)
    ref = y.double() + cs.double().exp()[..., None] * torch.einsum(
        "blhn,bhnp->blhp", C.double().expand(b, L, H, N), h_in.to(torch.bfloat16).double())
    yd = y.cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ssd.cp_correct(C.cuda(), cs.cuda(), h_in.cuda(), yd, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    err = (yd.double().cpu() - ref).abs().max() / ref.abs().max()
    assert err <= (2e-2 if out == torch.bfloat16 else 1e-4)
