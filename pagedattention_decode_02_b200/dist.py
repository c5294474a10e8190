"""Multi-GPU plumbing for the decode step: one process per GPU.

The decode step shards by sequence with no exchange on the data path: every
rank owns its own KV pool, block manager and sequences (data parallel over
independent requests).  The only cross-rank traffic is host-side bookkeeping:
splitting a global batch into per-rank shards and reducing the measured time
(max over ranks) and the work done (sum over ranks).  Works with any
``torch.distributed`` backend (NCCL over NVLink on GPUs, gloo on CPUs).
"""

from __future__ import annotations

import os
from datetime import timedelta
from typing import Sequence, Tuple


def rank_world() -> Tuple[int, int, int]:
    """(rank, world_size, local_rank) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: float = 120.0, device=None) -> None:
    """Join the process group (no-op for a single process)."""
    import torch.distributed as dist
    _, world, _ = rank_world()
    if world <= 1 or dist.is_initialized():
        return
    kw = {"timeout": timedelta(seconds=timeout_s)}
    if device is not None and backend == "nccl":
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def shard_bounds(n_items: int, rank: int, world: int) -> Tuple[int, int]:
    """[begin, end) of rank's contiguous share of n_items; shares differ by at
    most one item and cover every item exactly once."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(n_items, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def shard_sequences(seq_ids: Sequence[int], rank: int, world: int):
    b, e = shard_bounds(len(seq_ids), rank, world)
    return list(seq_ids[b:e])


def reduce_run(elapsed_ms: Sequence[float], work: Sequence[float], device=None):
    """Max over ranks of each elapsed time, sum over ranks of each work count.
    Single process: returned unchanged."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(x) for x in elapsed_ms], [float(x) for x in work]
    t = torch.tensor(list(elapsed_ms), dtype=torch.float64, device=device)
    w = torch.tensor(list(work), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(w, op=dist.ReduceOp.SUM)
    return [float(x) for x in t.cpu()], [float(x) for x in w.cpu()]


def barrier() -> None:
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def finish() -> None:
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
