"""Oracle pins for the reference block manager (CPU only).

* a block-table walk worked by hand from the pages' rules (golden file);
* invariants the pages fix, over random and exhaustive op streams: waste below
  one block per sequence, refcount conservation, no block both free and
  referenced, copy-on-write leaves every other sharer's view unchanged,
  all-or-nothing failures.
"""

import itertools
import json
import os
import random

import numpy as np
import pytest

from oracle.allocator import AllocError, BlockManager
from oracle.engine import DecodeOracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def check_invariants(bm: BlockManager):
    bs = bm.block_size
    counts = [0] * bm.num_blocks
    for s, t in bm.tables.items():
        n = bm.lengths[s]
        assert len(t) == -(-n // bs), "a block is taken only when the last one is full"
        assert 0 <= len(t) * bs - n <= bs - 1, "waste below one block"
        for b in t:
            counts[b] += 1
    assert counts == bm.refcount, "refcount = number of tables that hold the block"
    free = list(bm.free)
    assert len(set(free)) == len(free), "no block twice in the free queue"
    for b in range(bm.num_blocks):
        assert (b in set(free)) == (bm.refcount[b] == 0)
    assert len(free) + sum(1 for r in bm.refcount if r > 0) == bm.num_blocks


def test_worked_example():
    g = json.load(open(os.path.join(GOLD, "allocation_worked_example.json")))
    bm = BlockManager(g["num_blocks"], g["block_size"])
    for op in g["ops"]:
        try:
            if op["op"] == "alloc":
                r = bm.alloc(op["seq"], op["n"])
                assert r == op["slots"]
            elif op["op"] == "append":
                slot, src, dst = bm.append(op["seq"])
                assert slot == op["slot"]
                assert (None if src < 0 else [src, dst]) == op["cow"]
            elif op["op"] == "fork":
                bm.fork(op["parent"], op["child"])
            elif op["op"] == "free":
                bm.free_seq(op["seq"])
            assert "error" not in op
        except AllocError as e:
            assert e.status == op.get("error"), op
        check_invariants(bm)
    f = g["final"]
    assert {str(k): v for k, v in bm.tables.items()} == f["tables"]
    assert {str(k): v for k, v in bm.lengths.items()} == f["lengths"]
    assert list(bm.free) == f["free"]
    assert bm.refcount == f["refcount"]
    assert bm.cow_count == f["cow_count"]


def _random_ops(bm, rnd, n_ops, max_tokens):
    live = []
    next_id = 0
    for _ in range(n_ops):
        r = rnd.random()
        try:
            if r < 0.2 or not live:
                bm.alloc(next_id, rnd.randint(0, max_tokens))
                live.append(next_id)
                next_id += 1
            elif r < 0.55:
                s = rnd.choice(live)
                before = {o: list(bm.tables[o]) for o in live if o != s}
                bm.append(s)
                # copy-on-write never touches another sequence's table
                assert before == {o: bm.tables[o] for o in live if o != s}
            elif r < 0.7:
                k = rnd.randint(1, min(4, len(live)))
                bm.append_batch(rnd.sample(live, k))
            elif r < 0.85:
                bm.fork(rnd.choice(live), next_id)
                live.append(next_id)
                next_id += 1
            else:
                s = rnd.choice(live)
                bm.free_seq(s)
                live.remove(s)
        except AllocError as e:
            assert e.status == "NO_BLOCKS"
        check_invariants(bm)


@pytest.mark.parametrize("seed", range(20))
def test_random_op_streams_keep_invariants(seed):
    rnd = random.Random(seed)
    nb = rnd.randint(4, 40)
    bs = rnd.choice([1, 2, 3, 4, 8, 16])
    order = list(range(nb))
    rnd.shuffle(order)
    _random_ops(BlockManager(nb, bs, order), rnd, 300, 3 * bs)


def test_failures_change_nothing():
    bm = BlockManager(3, 2)
    bm.alloc(0, 3)
    bm.fork(0, 1)
    snap = bm._snapshot()
    with pytest.raises(AllocError) as e:
        bm.alloc(2, 5)
    assert e.value.status == "NO_BLOCKS"
    # batch: seq 0 copies (takes the last free block), seq 1 then writes in
    # place (refcount back to 1), the second append of seq 0 needs a fresh
    # block -> NO_BLOCKS, and the whole batch is undone
    with pytest.raises(AllocError):
        bm.append_batch([0, 1, 0, 0])
    assert (list(bm.free), bm.refcount, bm.tables, bm.lengths, bm.cow_count) == \
        (list(snap[0]), snap[1], snap[2], snap[3], snap[4])
    for bad in (lambda: bm.append(7), lambda: bm.free_seq(7), lambda: bm.fork(7, 8)):
        with pytest.raises(AllocError) as e:
            bad()
        assert e.value.status == "UNKNOWN_SEQ"
    with pytest.raises(AllocError) as e:
        bm.fork(0, 1)
    assert e.value.status == "SEQ_EXISTS"


def test_four_sharers_copy_three_times():
    # three of four sharers copy the partial last block; the fourth writes in
    # place; full shared blocks stay shared
    bm = BlockManager(16, 4)
    bm.alloc(0, 10)            # blocks 0,1 full, block 2 holds 2
    for c in (1, 2, 3):
        bm.fork(0, c)
    assert bm.refcount[:3] == [4, 4, 4]
    slots, pairs = bm.append_batch([0, 1, 2, 3])
    assert pairs == [(2, 3), (2, 4), (2, 5)]
    assert slots == [3 * 4 + 2, 4 * 4 + 2, 5 * 4 + 2, 2 * 4 + 2]
    assert bm.refcount[:6] == [4, 4, 1, 1, 1, 1]
    assert [bm.tables[s][:2] for s in range(4)] == [[0, 1]] * 4
    check_invariants(bm)


def test_full_shared_last_block_takes_fresh_block_no_copy():
    bm = BlockManager(8, 4)
    bm.alloc(0, 8)
    bm.fork(0, 1)
    slots, pairs = bm.append_batch([0, 1])
    assert pairs == []
    assert bm.tables[0] == [0, 1, 2] and bm.tables[1] == [0, 1, 3]
    assert bm.refcount[:4] == [2, 2, 1, 1]


def test_exhaustive_short_op_sequences():
    # every sequence of up to 4 ops over 2 sequence ids on a pool of 3 blocks
    # of 2: invariants hold and failures leave the state unchanged
    ops = [("alloc", 0, 1), ("alloc", 0, 3), ("alloc", 1, 2), ("append", 0), ("append", 1),
           ("fork", 0, 1), ("fork", 1, 0), ("free", 0), ("free", 1), ("batch", (0, 1))]
    n = 0
    for length in range(1, 5):
        for seq in itertools.product(ops, repeat=length):
            bm = BlockManager(3, 2)
            for op in seq:
                snap = bm._snapshot()
                try:
                    if op[0] == "alloc":
                        bm.alloc(op[1], op[2])
                    elif op[0] == "append":
                        bm.append(op[1])
                    elif op[0] == "fork":
                        bm.fork(op[1], op[2])
                    elif op[0] == "free":
                        bm.free_seq(op[1])
                    else:
                        bm.append_batch(op[1])
                except AllocError:
                    assert (list(bm.free), bm.refcount, bm.tables, bm.lengths) == \
                        (list(snap[0]), snap[1], snap[2], snap[3])
                check_invariants(bm)
                n += 1
    assert n > 30000


def test_cow_leaves_sharers_views_unchanged():
    # the data side: after every step every sequence's rows, read through its
    # own table from a pool image, equal its own history
    rnd = np.random.default_rng(3)
    bs, h, d = 4, 1, 4
    orc = DecodeOracle(64, bs, h, d, "f32", order=rnd.permutation(64))
    pool = np.zeros((64, h, bs, d), np.float32)

    def scatter(slots, rows):
        for sl, r in zip(slots, rows):
            pool[sl // bs, :, sl % bs, :] = r

    k = rnd.standard_normal((10, h, d)).astype(np.float32)
    scatter(orc.admit(0, k, k, "f32"), k)
    for c in (1, 2, 3):
        orc.fork(0, c)
    seqs = [0, 1, 2, 3]
    from oracle.engine import gather_rows
    for step in range(9):
        kn = rnd.standard_normal((4, h, d)).astype(np.float32)
        before = {s: gather_rows(pool, orc.bm.tables[s], orc.bm.lengths[s], bs).copy() for s in seqs}
        slots, pairs = orc.append(seqs, kn, kn, "f32")
        for src, dst in pairs:       # copy whole block, then write
            pool[dst] = pool[src]
        scatter(slots, kn)
        for i, s in enumerate(seqs):
            got = gather_rows(pool, orc.bm.tables[s], orc.bm.lengths[s], bs)
            assert np.array_equal(got, orc.history(s)[0])
            assert np.array_equal(got[:-1], before[s])
