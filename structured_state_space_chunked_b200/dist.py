"""Multi-process plumbing for running the SSD forward on several GPUs.

The forward pass partitions cleanly: documents (batch rows, or packed documents)
and heads are independent, so ranks need no data-path collective.  A global
batch is split into contiguous document ranges, one per rank, and every rank
runs ``ssd_forward`` on its range with its own handle.  The only collectives
are for coordination: a barrier around timed regions and a max over ranks of
the measured time.  One process per GPU; rank/world come from the usual
``RANK``/``WORLD_SIZE``/``LOCAL_RANK`` environment of ``torchrun``.
"""

from __future__ import annotations

import datetime
import os
from typing import Optional, Tuple

import torch
import torch.distributed as dist


def env_ranks() -> Tuple[int, int, int]:
    """(rank, world_size, local_rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: float = 120.0, device: Optional[torch.device] = None):
    """Join the process group when WORLD_SIZE > 1; returns the group module or None."""
    rank, world, _ = env_ranks()
    if world <= 1:
        return None
    kw = {}
    if backend == "nccl" and device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return dist


def shard_range(n: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous [start, stop) share of n independent items for `rank` of `world`.

    Shares differ by at most one item and cover 0..n-1 exactly once.
    """
    if world <= 0 or not (0 <= rank < world):
        raise ValueError("bad rank/world")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def shard_documents(cu_seqlens, world: int, rank: int):
    """This rank's documents of a packed row: (token_start, token_stop, local cu_seqlens).

    Documents are split into contiguous ranges balanced by document count; the
    local cu_seqlens is rebased to start at 0.
    """
    import numpy as np

    cu = np.asarray(cu_seqlens, dtype=np.int64)
    d0, d1 = shard_range(len(cu) - 1, world, rank)
    t0, t1 = int(cu[d0]), int(cu[d1])
    return t0, t1, (cu[d0:d1 + 1] - t0).astype(np.int32)


def barrier(group=None, device_sync: bool = True) -> None:
    if group is not None:
        group.barrier()
    if device_sync and torch.cuda.is_available():
        torch.cuda.synchronize()


def max_over_ranks(value: float, group=None, device: Optional[torch.device] = None) -> float:
    """Maximum of a per-rank scalar over all ranks (identity without a group)."""
    if group is None:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    group.all_reduce(t, op=group.ReduceOp.MAX)
    return float(t.item())


class _CudaOps:
    """The device steps of a context-parallel rank, on this library's kernels."""

    def __init__(self, handle):
        self.h = handle

    def forward(self, x, dt, A, B, C, D, dt_bias, chunk_size):
        return self.h.forward(x, dt, A, B, C, D, dt_bias, chunk_size, None, None)

    def logdecay(self, dt, A, dt_bias, x, B):
        from . import ssd
        return ssd.cp_logdecay(dt, A, dt_bias, headdim=x.shape[3], dstate=B.shape[3],
                               ngroups=B.shape[2])

    def combine(self, rank, S_all, ld_all, init, dt):
        from . import ssd
        return ssd.cp_combine(rank, S_all, ld_all, init, dt_dtype=dt.dtype)

    def correct(self, C, cs, h_in, y):
        from . import ssd
        return ssd.cp_correct(C, cs, h_in, y)


def context_parallel_forward(x, dt, A, B, C, D=None, dt_bias=None, chunk_size=256,
                             initial_states=None, group=None, handle=None, ops=None):
    """Chunked SSD forward over a sequence whose tokens are cut across the ranks.

    Every rank holds the same batch rows; rank r holds its consecutive slice of
    the tokens (x [b, L_r, H, P], dt [b, L_r, H], B/C [b, L_r, G, N]); slices go in
    rank order.  ``initial_states`` is the state before the whole sequence (the
    same on every rank, or None).  Returns this rank's y and the state at the end
    of its slice (on the last rank: the final state of the sequence).

    The one exchange step is an all-gather of each rank's local final state
    (b·H·N·P fp32) and total log decay (b·H fp32) ("Transformers are SSMs",
    paperlayer.ai summary, §8.2); everything else runs on the rank's own data
    through ``ops`` (default: this library's kernels on ``handle``, a
    :class:`ssd.SSD` of the slice's shape).
    """
    rank = group.get_rank() if group is not None else 0
    world = group.get_world_size() if group is not None else 1
    ops = ops or _CudaOps(handle)
    y, s_local = ops.forward(x, dt, A, B, C, D, dt_bias, chunk_size)
    cs, ld = ops.logdecay(dt, A, dt_bias, x, B)
    if group is not None and world > 1:
        S_parts = [torch.empty_like(s_local) for _ in range(world)]
        ld_parts = [torch.empty_like(ld) for _ in range(world)]
        group.all_gather(S_parts, s_local.contiguous())
        group.all_gather(ld_parts, ld.contiguous())
        S_all, ld_all = torch.stack(S_parts), torch.stack(ld_parts)
    else:
        S_all, ld_all = s_local[None], ld[None]
    h_in, final = ops.combine(rank, S_all.contiguous(), ld_all.contiguous(), initial_states, dt)
    ops.correct(C, cs, h_in, y)
    return y, final
