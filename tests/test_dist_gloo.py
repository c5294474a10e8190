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


# ---------------------------------------------------------------------------
# the sequence-sharded layout itself: each rank owns an independent pool
# ---------------------------------------------------------------------------
ROUNDS = 40


def _sharded_worker(rank, world, port, out):
    """One rank: its shard of the OPT-13B-shaped batch on a pool of its own
    (host-only: the block manager alone), admitted and grown by ROUNDS decode
    rounds through the C ABI; an oracle allocator runs the same shard."""
    import numpy as np

    import pagedattention_decode_02_b200 as pk
    import workloads as wl
    from oracle.allocator import BlockManager

    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    pd.init("gloo", timeout_s=60)
    r, w, _ = pd.rank_world()
    cfg = wl.CONFIGS["opt13b"]
    lens = wl.history_lengths(cfg, 0)
    mine = pd.shard_sequences(list(range(cfg.batch)), r, w)
    nb = wl.pool_blocks(cfg, [lens[s] for s in mine], ROUNDS)
    order = wl.free_order(nb, 100 + r, cfg.permute)
    pool = pk.kv_pool_create(nb, cfg.block_size, cfg.n_kv_heads, cfg.head_dim, cfg.kv_dtype,
                             host_only=True)
    pk.bt_reset(pool, order)
    orc = BlockManager(nb, cfg.block_size, order)
    ok = True
    for s in mine:
        ok &= pk.bt_alloc(pool, s, int(lens[s])).tolist() == orc.alloc(s, int(lens[s]))
    for _ in range(ROUNDS):
        slots, src, dst = pk.bt_append_batch(pool, mine)
        o_slots, o_pairs = orc.append_batch(mine)
        ok &= slots.tolist() == o_slots and list(zip(src.tolist(), dst.tolist())) == o_pairs
    max_blocks = max(pk.bt_num_blocks(pool, s) for s in mine)
    tables, clens, fills = pk.bt_export(pool, mine, max_blocks)
    o_tables, o_lens, o_fills = orc.export(mine, max_blocks)
    ok &= tables.tolist() == o_tables and clens.tolist() == o_lens and fills.tolist() == o_fills
    st = pk.bt_stats(pool)
    ost = orc.stats()
    keys = ("used_blocks", "num_seqs", "stored_slots", "logical_tokens", "table_slots",
            "cow_count", "free_blocks")
    ok &= all(st[k] == ost[k] for k in keys)
    # the batch-wide counters: sums over the ranks' pools
    _, sums = pd.reduce_run([0.0], [float(st[k]) for k in keys[:-1]])
    pd.barrier()
    out[r] = (bool(ok), mine, sums)
    pool.close()
    pd.finish()


def test_two_ranks_own_independent_pools():
    import workloads as wl
    from oracle.allocator import BlockManager

    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_sharded_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    for r in range(world):
        assert out[r][0], f"rank {r}: tables, slots or stats differ from its oracle allocator"
    cfg = wl.CONFIGS["opt13b"]
    assert sorted(out[0][1] + out[1][1]) == list(range(cfg.batch))
    # one pool holding the whole batch gives the same batch-wide counters
    lens = wl.history_lengths(cfg, 0)
    nb = wl.pool_blocks(cfg, lens, ROUNDS)
    orc = BlockManager(nb, cfg.block_size, wl.free_order(nb, 0, cfg.permute))
    for s in range(cfg.batch):
        orc.alloc(s, int(lens[s]))
    for _ in range(ROUNDS):
        orc.append_batch(list(range(cfg.batch)))
    whole = orc.stats()
    keys = ("used_blocks", "num_seqs", "stored_slots", "logical_tokens", "table_slots",
            "cow_count")
    for r in range(world):
        assert out[r][2] == [float(whole[k]) for k in keys]
