"""The multi-rank path on CPU: two gloo ranks split a batch of independent
documents, each computes its share, and the shares together equal the
single-process result; the coordination collectives (barrier, max over ranks)
behave as the benchmark uses them."""

import json
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from structured_state_space_chunked_b200 import dist as sdist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("n,world", [(8, 2), (7, 2), (5, 3), (1, 4), (0, 2), (10, 1)])
def test_shard_range_partitions_exactly(n, world):
    got = []
    sizes = []
    for r in range(world):
        a, b = sdist.shard_range(n, world, r)
        got.extend(range(a, b))
        sizes.append(b - a)
    assert got == list(range(n))
    assert max(sizes) - min(sizes) <= 1


def test_shard_documents_rebases_cu_seqlens():
    cu = np.array([0, 5, 9, 20, 21, 30], dtype=np.int32)
    t0, t1, loc = sdist.shard_documents(cu, 2, 1)
    assert (t0, t1) == (20, 30)
    assert loc.tolist() == [0, 1, 10]
    t0, t1, loc = sdist.shard_documents(cu, 2, 0)
    assert (t0, t1) == (0, 20) and loc.tolist() == [0, 5, 9, 20]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import oracle
    from structured_state_space_chunked_b200 import dist as d
    from structured_state_space_chunked_b200 import inputs as I

    group = d.init("gloo", timeout_s=60)
    w = I.random_small(77, "fp32", 5, 40, 3, 4, 6, 1, 16, "normal0.1")
    inp = I.make_inputs(w)
    b0, b1 = d.shard_range(w.batch, world, rank)
    part = {k: (None if v is None else v[b0:b1]) for k, v in inp.items() if k != "cu_seqlens"}
    y, fin = oracle.oracle_forward(part["x"], part["dt"], inp["A"], part["B"], part["C"], inp["D"],
                                   inp["dt_bias"], part["initial_states"])
    gathered = [None] * world
    group.all_gather_object(gathered, (b0, b1, y.tolist(), fin.tolist()))
    d.barrier(group, device_sync=False)
    mx = d.max_over_ranks(10.0 + rank, group)
    if rank == 0:
        yf, ff = oracle.oracle_forward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                                       inp["dt_bias"], inp["initial_states"])
        ys = np.concatenate([np.asarray(g[2]) for g in gathered if g[1] > g[0]], axis=0)
        fs = np.concatenate([np.asarray(g[3]) for g in gathered if g[1] > g[0]], axis=0)
        res = dict(equal_y=bool(np.array_equal(ys, yf)), equal_f=bool(np.array_equal(fs, ff)),
                   max=mx, ranges=[(g[0], g[1]) for g in gathered])
        with open(os.path.join(out_dir, "res.json"), "w") as f:
            json.dump(res, f)
    group.destroy_process_group()


def test_two_gloo_ranks_split_a_batch(tmp_path):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = json.load(open(tmp_path / "res.json"))
    assert res["equal_y"] and res["equal_f"]
    assert res["max"] == 11.0
    assert res["ranges"] == [[0, 3], [3, 5]]


class _CpuOps:
    """Test-only float64 stand-ins for the device steps of a context-parallel rank
    (the collectives and their orchestration are the code under test)."""

    def forward(self, x, dt, A, B, C, D, dt_bias, chunk_size):
        import oracle
        y, fin = oracle.oracle_forward(x, dt, A, B, C, D, dt_bias, None)
        return torch.tensor(y), torch.tensor(fin)

    def logdecay(self, dt, A, dt_bias, x, B):
        la = np.logaddexp(0.0, dt.double().numpy() + dt_bias.double().numpy()[None, None, :])
        cs = np.cumsum(la * A.double().numpy()[None, None, :], axis=1)
        return torch.tensor(cs), torch.tensor(np.ascontiguousarray(cs[:, -1]))

    def combine(self, rank, S_all, ld_all, init, dt):
        S, ld = S_all.numpy(), ld_all.numpy()
        h = np.zeros(S.shape[1:]) if init is None else init.double().numpy().copy()
        for k in range(rank):
            h = np.exp(ld[k])[..., None, None] * h + S[k]
        return torch.tensor(h), torch.tensor(np.exp(ld[rank])[..., None, None] * h + S[rank])

    def correct(self, C, cs, h_in, y):
        H, G = y.shape[2], C.shape[2]
        Ch = C.double().numpy()[:, :, np.arange(H) // (H // G), :]        # [b, L, H, N]
        add = np.einsum("blhn,bhnp->blhp", Ch, h_in.numpy()) * np.exp(cs.numpy())[..., None]
        y += torch.tensor(add)
        return y


def _cp_rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import oracle
    from structured_state_space_chunked_b200 import dist as d
    from structured_state_space_chunked_b200 import inputs as I

    group = d.init("gloo", timeout_s=60)
    w = I.random_small(91, "fp32", 2, 42, 4, 3, 5, 2, 16, "normal0.1")
    inp = I.make_inputs(w)
    t0, t1 = d.shard_range(w.seqlen, world, rank)
    part = {k: inp[k][:, t0:t1].contiguous() for k in ("x", "dt", "B", "C")}
    y, fin = d.context_parallel_forward(part["x"], part["dt"], inp["A"], part["B"], part["C"],
                                        inp["D"], inp["dt_bias"], 16, inp["initial_states"],
                                        group=group, ops=_CpuOps())
    gathered = [None] * world
    group.all_gather_object(gathered, (t0, t1, y.numpy().tolist(), fin.numpy().tolist()))
    if rank == 0:
        yf, ff = oracle.oracle_forward(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                                       inp["dt_bias"], inp["initial_states"])
        ys = np.concatenate([np.asarray(g[2]) for g in gathered], axis=1)
        ey = float(np.max(np.abs(ys - yf)) / np.max(np.abs(yf)))
        ef = float(np.max(np.abs(np.asarray(gathered[-1][3]) - ff)) / np.max(np.abs(ff)))
        with open(os.path.join(out_dir, "cp.json"), "w") as f:
            json.dump(dict(ey=ey, ef=ef, ranges=[(g[0], g[1]) for g in gathered]), f)
    group.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_ranks_reproduce_the_whole_sequence(tmp_path, world):
    # each rank holds a slice of the tokens; after the all-gather of local final
    # states and log decays, the ranks' outputs together equal one run over the
    # whole sequence, and the last rank holds its final state
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_cp_rank_main, args=(r, world, port, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = json.load(open(tmp_path / "cp.json"))
    assert res["ey"] < 1e-10 and res["ef"] < 1e-10, res
    assert res["ranges"][0][0] == 0 and res["ranges"][-1][1] == 42
