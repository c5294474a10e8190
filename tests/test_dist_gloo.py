"""The N > 1 host path on CPU: two gloo ranks split a batch and reduce the
measured run (max of times, sum of work), as bench.py does over NCCL."""

import os
import socket

import pytest
import torch.multiprocessing as mp

from pagedattention_decode_02_b200 import dist as pd


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    pd.init("gloo", timeout_s=30)
    r, w, _ = pd.rank_world()
    mine = pd.shard_sequences(list(range(30)), r, w)
    times, work = pd.reduce_run([10.0 + r, 1.0 * r], [float(len(mine)), 100.0])
    pd.barrier()
    out[r] = (mine, times, work)
    pd.finish()


def test_two_gloo_ranks_shard_and_reduce():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    shards = [out[r][0] for r in range(world)]
    assert sorted(shards[0] + shards[1]) == list(range(30))      # every sequence exactly once
    for r in range(world):
        _, times, work = out[r]
        assert times == [11.0, 1.0]                               # max over ranks
        assert work == [30.0, 200.0]                              # sum over ranks


@pytest.mark.parametrize("n,world", [(30, 1), (30, 4), (7, 8), (0, 3), (128, 8)])
def test_shard_bounds_cover_exactly_once(n, world):
    seen = []
    sizes = []
    for r in range(world):
        b, e = pd.shard_bounds(n, r, world)
        seen.extend(range(b, e))
        sizes.append(e - b)
    assert seen == list(range(n))
    assert max(sizes) - min(sizes) <= 1
