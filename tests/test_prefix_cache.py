"""Automatic prefix caching (CPU): the reference allocator against a
hand-worked walk and the published FNV-1a test vectors, and the C++ block
manager against the reference allocator bit-exactly over random admission
streams with shared prompt prefixes."""

import json
import os
import random

import pytest

import pagedattention_decode_02_b200 as pk
from oracle.allocator import AllocError, BlockManager, block_key, fnv1a64

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_fnv1a64_published_vectors():
    # the FNV reference test vectors for FNV-1a, 64 bit
    assert fnv1a64(b"") == 0xCBF29CE484222325
    assert fnv1a64(b"a") == 0xAF63DC4C8601EC8C
    assert fnv1a64(b"foobar") == 0x85944171F73967E8


def test_block_key_chains_over_the_prefix():
    a = block_key(0, [1, 2])
    assert block_key(a, [3, 4]) != block_key(0, [3, 4])        # position matters
    assert block_key(0, [1, 2]) == a
    assert block_key(0, [2, 1]) != a


def _apply(mgr, op, native=False):
    if op["op"] == "alloc_prefix":
        if native:
            slots, cached = pk.bt_alloc_prefix(mgr, op["seq"], op["tokens"])
            return slots.tolist(), cached
        return mgr.alloc_prefix(op["seq"], op["tokens"])
    if op["op"] == "alloc":
        return (pk.bt_alloc(mgr, op["seq"], op["n"]).tolist() if native
                else mgr.alloc(op["seq"], op["n"]))
    if op["op"] == "free":
        return pk.bt_free(mgr, op["seq"]) if native else mgr.free_seq(op["seq"])
    raise ValueError(op)


@pytest.mark.parametrize("native", [False, True])
def test_worked_example(native):
    g = json.load(open(os.path.join(GOLD, "prefix_cache_worked_example.json")))
    if native:
        mgr = pk.kv_pool_create(g["num_blocks"], g["block_size"], 1, 32, "f32", host_only=True)
        pk.bt_set_prefix_caching(mgr, True)
    else:
        mgr = BlockManager(g["num_blocks"], g["block_size"])
        mgr.set_prefix_caching(True)
    for op in g["ops"]:
        try:
            r = _apply(mgr, op, native)
            assert "error" not in op
        except (AllocError, pk.PagedKVError) as e:
            status = e.status if isinstance(e, AllocError) else e.name
            assert status == op["error"]
            continue
        if op["op"] == "alloc_prefix":
            assert list(r[0]) == op["slots"] and r[1] == op["cached"]
        if "free_after" in op:
            free = pk.bt_free_queue(mgr).tolist() if native else list(mgr.free)
            assert free == op["free_after"]
    f = g["final"]
    if native:
        assert pk.bt_free_queue(mgr).tolist() == f["free"]
        assert [pk.bt_refcount(mgr, b) for b in range(g["num_blocks"])] == f["refcount"]
        st = pk.bt_stats(mgr)
    else:
        assert list(mgr.free) == f["free"]
        assert mgr.refcount == f["refcount"]
        st = mgr.stats()
    assert st["prefix_hit_tokens"] == f["prefix_hit_tokens"]
    assert st["cached_blocks"] == f["cached_blocks"]


def _prompt(rnd, prefixes, bs):
    base = list(rnd.choice(prefixes))
    cut = rnd.randint(0, len(base))
    tail = [rnd.randint(0, 3) for _ in range(rnd.randint(0, 3 * bs))]
    return base[:cut] + tail


@pytest.mark.parametrize("seed", range(20))
def test_random_streams_native_matches_reference(seed):
    rnd = random.Random(seed)
    nb = rnd.randint(4, 40)
    bs = rnd.choice([1, 2, 3, 4, 8])
    order = list(range(nb))
    rnd.shuffle(order)
    prefixes = [[rnd.randint(0, 3) for _ in range(rnd.randint(1, 5 * bs))] for _ in range(3)]
    p = pk.kv_pool_create(nb, bs, 1, 32, "f16", host_only=True)
    pk.bt_reset(p, order)
    pk.bt_set_prefix_caching(p, True)
    ref = BlockManager(nb, bs, order)
    ref.set_prefix_caching(True)
    live, nxt = [], 0

    def both(fa, fb):
        try:
            a = fa()
        except pk.PagedKVError as e:
            a = e.name
        try:
            b = fb()
        except AllocError as e:
            b = e.status
        return a, b

    for _ in range(250):
        r = rnd.random()
        if r < 0.35 or not live:
            toks = _prompt(rnd, prefixes, bs)
            a, b = both(lambda: pk.bt_alloc_prefix(p, nxt, toks), lambda: ref.alloc_prefix(nxt, toks))
            if isinstance(b, str):
                assert a == b
            else:
                assert a[0].tolist() == b[0] and a[1] == b[1]
                live.append(nxt)
                # the reused blocks hold exactly this prompt's leading tokens
                for i in range(b[1] // bs):
                    blk = ref.tables[nxt][i]
                    assert ref.registered[blk][1] == toks[i * bs:(i + 1) * bs]
            nxt += 1
        elif r < 0.6:
            ids = [rnd.choice(live) for _ in range(rnd.randint(1, 3))]
            a, b = both(lambda: pk.bt_append_batch(p, ids), lambda: ref.append_batch(ids))
            if isinstance(b, str):
                assert a == b
            else:
                assert a[0].tolist() == b[0]
        elif r < 0.7:
            s = rnd.choice(live)
            a, b = both(lambda: pk.bt_fork(p, s, nxt), lambda: ref.fork(s, nxt))
            if not isinstance(b, str):
                live.append(nxt)
            nxt += 1
        else:
            s = rnd.choice(live)
            pk.bt_free(p, s)
            ref.free_seq(s)
            live.remove(s)
        assert pk.bt_free_queue(p).tolist() == list(ref.free)
        assert [pk.bt_refcount(p, b) for b in range(nb)] == ref.refcount
        st, rs = pk.bt_stats(p), ref.stats()
        for k in ("prefix_hit_tokens", "cached_blocks", "free_blocks", "logical_tokens"):
            assert st[k] == rs[k], k


def test_caching_off_behaves_like_alloc():
    p = pk.kv_pool_create(8, 2, 1, 32, "f32", host_only=True)
    s1, c1 = pk.bt_alloc_prefix(p, 0, [1, 2, 3, 4])
    s2, c2 = pk.bt_alloc_prefix(p, 1, [1, 2, 3, 4])
    assert c1 == c2 == 0 and s1.tolist() == [0, 1, 2, 3] and s2.tolist() == [4, 5, 6, 7]
    pk.bt_set_prefix_caching(p, True)
    pk.bt_alloc_prefix(p, 2, [5, 6, 7, 8])
    pk.bt_free(p, 0)
    pk.bt_free(p, 1)
    _, c3 = pk.bt_alloc_prefix(p, 3, [5, 6, 7, 8, 1])
    assert c3 == 4
    pk.bt_set_prefix_caching(p, False)                  # forgets every registration
    assert pk.bt_stats(p)["cached_blocks"] == 0
