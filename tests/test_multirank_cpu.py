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
