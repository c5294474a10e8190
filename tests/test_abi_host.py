"""The C ABI library on the CPU: it loads, exports every function the header
declares, and its host block manager (a host-only pool) matches the oracle's
reference allocator bit-exactly over worked, random and failing op streams."""

import json
import os
import random
import re
import subprocess

import numpy as np
import pytest

import pagedattention_decode_02_b200 as pk
from oracle.allocator import AllocError, BlockManager

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedkv.h")
GOLD = os.path.join(os.path.dirname(__file__), "golden")

STATUS = {"NO_BLOCKS": pk.PKV_ERR_NO_BLOCKS, "UNKNOWN_SEQ": pk.PKV_ERR_UNKNOWN_SEQ,
          "SEQ_EXISTS": pk.PKV_ERR_SEQ_EXISTS, "INVALID_ARG": pk.PKV_ERR_INVALID_ARG}


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w \*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("kv_pool_create", "bt_alloc", "bt_append", "bt_fork", "bt_free", "kv_append",
                 "paged_decode_attention", "block_copy"):
        assert want in names
    assert len(names) >= 20


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", pk.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(pk._lib, n)
    assert set(pk.EXPORTED) == set(declared_functions())


def test_status_strings():
    assert pk.pkv_status_str(pk.PKV_OK) == "OK"
    assert pk.pkv_status_str(pk.PKV_ERR_NO_BLOCKS) == "NO_BLOCKS"
    assert pk.pkv_status_str(99) == "UNKNOWN_STATUS"


def test_pool_size_query_and_argument_checks():
    assert pk.kv_pool_bytes(10, 16, 40, 128, "f16") == 10 * 16 * 40 * 128 * 2
    assert pk.kv_pool_bytes(3, 4, 1, 32, "fp8") == 3 * 4 * 32
    for bad in [(0, 16, 1, 128, "f16"), (4, 0, 1, 128, "f16"), (4, 16, 0, 128, "f16"),
                (4, 16, 1, 96, "f16")]:
        with pytest.raises(pk.PagedKVError) as e:
            pk.kv_pool_create(*bad, host_only=True)
        assert e.value.status == pk.PKV_ERR_INVALID_ARG
    with pytest.raises(pk.PagedKVError):
        pk.kv_pool_create(4, 16, 1, 128, "fp8", k_scale=0.0, host_only=True)


def test_host_only_pool_refuses_device_calls():
    p = pk.kv_pool_create(4, 4, 1, 32, "f32", host_only=True)
    st = pk._lib.kv_append(p.handle, None, 1, None, None, pk.PKV_F32, None)
    assert st == pk.PKV_ERR_INVALID_ARG
    st = pk._lib.paged_decode_attention(p.handle, None, pk.PKV_F32, None, 1, None, 1, 1, 1.0,
                                        None, None, 0, None)
    assert st == pk.PKV_ERR_INVALID_ARG


def test_worked_example_matches_golden():
    g = json.load(open(os.path.join(GOLD, "allocation_worked_example.json")))
    p = pk.kv_pool_create(g["num_blocks"], g["block_size"], 1, 32, "f32", host_only=True)
    for op in g["ops"]:
        try:
            if op["op"] == "alloc":
                assert list(pk.bt_alloc(p, op["seq"], op["n"])) == op["slots"]
            elif op["op"] == "append":
                slot, src, dst = pk.bt_append(p, op["seq"])
                assert slot == op["slot"]
                assert (None if src < 0 else [src, dst]) == op["cow"]
            elif op["op"] == "fork":
                pk.bt_fork(p, op["parent"], op["child"])
            elif op["op"] == "free":
                pk.bt_free(p, op["seq"])
            assert "error" not in op
        except pk.PagedKVError as e:
            assert e.status == STATUS[op["error"]], op
    f = g["final"]
    for s, t in f["tables"].items():
        tables, lens, fills = pk.bt_export(p, [int(s)], 4)
        assert list(tables[0][: len(t)]) == t and all(tables[0][len(t):] == -1)
        assert lens[0] == f["lengths"][s]
    assert list(pk.bt_free_queue(p)) == f["free"]
    assert [pk.bt_refcount(p, b) for b in range(g["num_blocks"])] == f["refcount"]
    assert pk.bt_stats(p)["cow_count"] == f["cow_count"]


def _compare(p, bm: BlockManager, live):
    ids = sorted(live)
    if ids:
        mb = max(1, max(len(bm.tables[s]) for s in ids))
        t, l, f = pk.bt_export(p, ids, mb)
        rt, rl, rf = bm.export(ids, mb)
        assert t.tolist() == rt and l.tolist() == rl and f.tolist() == rf
    assert pk.bt_free_queue(p).tolist() == list(bm.free)
    st = pk.bt_stats(p)
    rs = bm.stats()
    for k in ("free_blocks", "used_blocks", "num_seqs", "stored_slots", "logical_tokens",
              "table_slots", "cow_count"):
        assert st[k] == rs[k], k


def _status_of(fn):
    try:
        return fn(), None
    except pk.PagedKVError as e:
        return None, e.name
    except AllocError as e:
        return None, e.status


@pytest.mark.parametrize("seed", range(25))
def test_random_streams_bit_exact_vs_oracle(seed):
    rnd = random.Random(1000 + seed)
    nb = rnd.randint(1, 48)
    bs = rnd.choice([1, 2, 3, 4, 5, 8, 16, 32])
    order = list(range(nb))
    rnd.shuffle(order)
    p = pk.kv_pool_create(nb, bs, 2, 64, "f16", host_only=True)
    pk.bt_reset(p, order)
    bm = BlockManager(nb, bs, order)
    live = set()
    nxt = 0
    for _ in range(400):
        r = rnd.random()
        if r < 0.18 or not live:
            n = rnd.randint(0, 4 * bs)
            a, ea = _status_of(lambda: pk.bt_alloc(p, nxt, n))
            b, eb = _status_of(lambda: bm.alloc(nxt, n))
            assert ea == eb
            if ea is None:
                assert a.tolist() == b
                live.add(nxt)
            nxt += 1
        elif r < 0.5:
            s = rnd.choice(sorted(live) + [nxt + 5])   # sometimes unknown
            a, ea = _status_of(lambda: pk.bt_append(p, s))
            b, eb = _status_of(lambda: bm.append(s))
            assert ea == eb and a == b
        elif r < 0.68:
            k = rnd.randint(1, min(6, len(live)))
            ids = [rnd.choice(sorted(live)) for _ in range(k)]   # repeats allowed
            a, ea = _status_of(lambda: pk.bt_append_batch(p, ids))
            b, eb = _status_of(lambda: bm.append_batch(ids))
            assert ea == eb
            if ea is None:
                assert a[0].tolist() == b[0]
                assert list(zip(a[1].tolist(), a[2].tolist())) == b[1]
        elif r < 0.82:
            par = rnd.choice(sorted(live))
            child = rnd.choice([nxt, par])                       # sometimes existing
            a, ea = _status_of(lambda: pk.bt_fork(p, par, child))
            b, eb = _status_of(lambda: bm.fork(par, child))
            assert ea == eb
            if ea is None:
                live.add(child)
                nxt += 1
        else:
            s = rnd.choice(sorted(live))
            pk.bt_free(p, s)
            bm.free_seq(s)
            live.discard(s)
        _compare(p, bm, live)


def test_reset_rejects_non_permutations():
    p = pk.kv_pool_create(4, 4, 1, 32, "f32", host_only=True)
    for bad in ([0, 1, 2, 2], [0, 1, 2, 4], [-1, 0, 1, 2]):
        with pytest.raises(pk.PagedKVError) as e:
            pk.bt_reset(p, bad)
        assert e.value.status == pk.PKV_ERR_INVALID_ARG
    pk.bt_reset(p, [3, 2, 1, 0])
    assert pk.bt_alloc(p, 0, 5).tolist() == [12, 13, 14, 15, 8]


def test_export_checks_capacity_and_writes_nothing_on_error():
    p = pk.kv_pool_create(8, 2, 1, 32, "f32", host_only=True)
    pk.bt_alloc(p, 0, 5)
    with pytest.raises(pk.PagedKVError) as e:
        pk.bt_export(p, [0], 2)
    assert e.value.status == pk.PKV_ERR_INVALID_ARG
    with pytest.raises(pk.PagedKVError) as e:
        pk.bt_export(p, [0, 9], 3)
    assert e.value.status == pk.PKV_ERR_UNKNOWN_SEQ


def test_config_batches_allocate_like_the_oracle():
    # the five workloads' admissions: identical tables, slots and free queues
    import workloads as wl
    for name in ("toy", "opt13b", "llama2_70b", "fp8"):
        cfg = wl.CONFIGS[name]
        if name == "fp8":
            cfg = cfg.with_block_size(4)
        lens = wl.history_lengths(cfg, 0)
        nb = wl.pool_blocks(cfg, lens)
        order = wl.free_order(nb, 0, cfg.permute)
        p = pk.kv_pool_create(nb, cfg.block_size, cfg.n_kv_heads, cfg.head_dim, cfg.kv_dtype,
                              host_only=True)
        pk.bt_reset(p, order)
        bm = BlockManager(nb, cfg.block_size, order)
        for i, n in enumerate(lens):
            assert pk.bt_alloc(p, i, int(n)).tolist() == bm.alloc(i, int(n))
        a = pk.bt_append_batch(p, list(range(len(lens))))
        b = bm.append_batch(list(range(len(lens))))
        assert a[0].tolist() == b[0]
        _compare(p, bm, set(range(len(lens))))


@pytest.mark.parametrize("bs", [1, 2, 4, 8, 16, 32, 64])
def test_utilisation_readout_fp8_sweep(bs):
    # bt_stats after admitting the FP8 sweep's 128 sequences and one append:
    # logical tokens / reserved slots, exactly the closed form over the same
    # lengths (a block is taken only when the last one is full)
    from fractions import Fraction
    from oracle.closed_forms import max_reservation_utilisation, utilisation
    import workloads as wl
    cfg = wl.CONFIGS["fp8"].with_block_size(bs)
    lens = wl.history_lengths(cfg, 0)
    nb = wl.pool_blocks(cfg, lens)
    p = pk.kv_pool_create(nb, bs, cfg.n_kv_heads, cfg.head_dim, "fp8", 0.01, 0.01, host_only=True)
    pk.bt_reset(p, wl.free_order(nb, 0, True))
    for i, n in enumerate(lens):
        pk.bt_alloc(p, i, int(n))
    pk.bt_append_batch(p, list(range(len(lens))))
    st = pk.bt_stats(p)
    ctx = [int(n) + 1 for n in lens]
    assert Fraction(st["logical_tokens"], st["table_slots"]) == utilisation(ctx, bs)
    assert st["stored_slots"] == st["logical_tokens"]          # nothing shared
    if bs == 1:
        assert st["logical_tokens"] == st["table_slots"]
    # reserving the maximum length (2,048 + 1) up front stores about half as much
    assert float(max_reservation_utilisation(ctx, 2049)) < 0.55


def test_guard_check_on_a_host_only_pool():
    # no device buffers, no guards: reported intact without touching a device
    pool = pk.kv_pool_create(16, 4, 2, 64, "f16", host_only=True)
    assert pk.kv_pool_check_guards(pool)
    pool.close()
    st = pk._lib.kv_pool_check_guards(None, None)
    assert st == pk.PKV_ERR_INVALID_ARG
