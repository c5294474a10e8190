"""GPU parity of the decode-step runtime (pkv_decode_step): host bookkeeping,
packed table upload, copy-on-write, append and attention in one call per
round, checked against the oracle round by round."""

import numpy as np
import pytest
import torch

import pagedattention_decode_02_b200 as pk
import workloads as wl
from paged_harness import (check_pool_bytes, compare_out, setup_config, step_inputs, to_torch,
                           from_torch)
from oracle.numerics import to_f64

pytestmark = pytest.mark.gpu


def run_rounds(cfg, side, steps, heads=None, partition=0, kernel=0):
    seqs = np.asarray(side.seqs, dtype=np.int64)
    max_blocks = max(len(side.orc.bm.tables[s]) for s in side.seqs) + steps // cfg.block_size + 2
    step = pk.Step(side.pool, len(seqs), max_blocks, cfg.n_q_heads, cfg.q_dtype, partition, kernel)
    out = torch.empty((len(seqs), cfg.n_q_heads, cfg.head_dim), device="cuda",
                      dtype={"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[cfg.q_dtype])
    worst = 0.0
    launches = []
    for t in range(steps):
        q, kn, vn = step_inputs(side, seqs, t)
        pk.pkv_decode_step(step, seqs, to_torch(q, cfg.q_dtype), to_torch(kn, cfg.q_dtype),
                           to_torch(vn, cfg.q_dtype), cfg.scale, out)
        launches.append(step.last_launches)
        side.orc.append(list(seqs), kn, vn, cfg.q_dtype)
        ref = side.orc.attend(list(seqs), q, cfg.q_dtype, cfg.scale, heads=heads)
        torch.cuda.synchronize()
        gpu = to_f64(from_torch(out, cfg.q_dtype), cfg.q_dtype)
        worst = max(worst, compare_out(gpu, ref, cfg.q_dtype if cfg.kv_dtype != "fp8" else "fp8", heads))
    assert pk.pkv_device_error(side.pool) == 0
    return worst, launches


def test_step_runtime_toy():
    cfg = wl.CONFIGS["toy"]
    side = setup_config(cfg, growth=8)
    run_rounds(cfg, side, 8)
    check_pool_bytes(side)


def test_step_runtime_copy_on_write():
    cfg = wl.CONFIGS["falcon7b"]
    import dataclasses
    cfg = dataclasses.replace(cfg, batch=8)          # 2 prompts x 4 samples
    side = setup_config(cfg, variant="b", growth=20)
    _, launches = run_rounds(cfg, side, 20, heads=[0, 35, 70])
    check_pool_bytes(side)
    assert launches[0] >= 2                           # (copy +) append + decode
    assert pk.bt_stats(side.pool)["cow_count"] == 2 * 3


def test_step_runtime_split_and_profile():
    cfg = wl.CONFIGS["opt13b"]
    import dataclasses
    cfg = dataclasses.replace(cfg, n_q_heads=4, n_kv_heads=4, batch=6, lengths=("uniform", 500, 1500),
                              min_pool_blocks=0)
    side = setup_config(cfg, growth=4)
    seqs = np.asarray(side.seqs, dtype=np.int64)
    step = pk.Step(side.pool, len(seqs), 128, cfg.n_q_heads, cfg.q_dtype, 0, 0)
    pk.pkv_step_profile(step, 4)
    out = torch.empty((len(seqs), 4, 128), device="cuda", dtype=torch.float16)
    for t in range(3):
        q, kn, vn = step_inputs(side, seqs, t)
        pk.pkv_decode_step(step, seqs, to_torch(q, "f16"), to_torch(kn, "f16"), to_torch(vn, "f16"),
                           cfg.scale, out)
        side.orc.append(list(seqs), kn, vn, "f16")
        # prologue (append) + decode + merge (the one-head CUDA-core kernel
        # leaves the merge to its own kernel)
        assert step.last_launches == 3
    ref = side.orc.attend(list(seqs), q, "f16", cfg.scale)
    torch.cuda.synchronize()
    compare_out(to_f64(from_torch(out, "f16"), "f16"), ref, "f16")
    pro, dec, mer = pk.pkv_step_profile_read(step, 4)
    assert len(dec) == 3 and np.all(dec > 0) and np.all(pro > 0) and np.all(mer >= 0)


@pytest.mark.parametrize("kernel", [pk.PKV_KERNEL_SIMT_TMA, pk.PKV_KERNEL_SIMT_BULK,
                                    pk.PKV_KERNEL_TENSOR])
def test_step_runtime_split_merge_every_kernel(kernel):
    # many rounds with split contexts: the in-kernel merge counters must come
    # back to zero after every launch (else later rounds merge too early)
    import dataclasses
    hkv = 2 if kernel == pk.PKV_KERNEL_TENSOR else 4
    cfg = dataclasses.replace(wl.CONFIGS["opt13b"], n_q_heads=4, n_kv_heads=hkv, batch=5,
                              lengths=("uniform", 100, 1200), min_pool_blocks=0)
    side = setup_config(cfg, growth=12)
    worst, launches = run_rounds(cfg, side, 12, partition=64, kernel=kernel)
    assert launches[-1] == (2 if kernel == pk.PKV_KERNEL_TENSOR else 3)


@pytest.mark.parametrize("base,hq,hkv,bs,expect", [
    ("opt13b", 4, 4, 16, pk.PKV_KERNEL_SIMT_TMA),      # MHA f16
    ("llama2_70b", 16, 2, 16, pk.PKV_KERNEL_TENSOR),   # GQA bf16, 8 heads per KV head
    ("falcon7b", 71, 1, 16, pk.PKV_KERNEL_LEAN),       # MQA, 71 heads per KV head
    ("fp8", 4, 4, 16, pk.PKV_KERNEL_TENSOR),           # FP8 MHA: codes converted for the tensor cores
    ("fp8", 4, 4, 1, pk.PKV_KERNEL_SIMT_TMA),          # ... but not with one token per block
    ("fp8_gqa", 16, 2, 16, pk.PKV_KERNEL_TENSOR),      # FP8 GQA on the tensor cores
])
def test_step_runtime_automatic_kernel(base, hq, hkv, bs, expect):
    import dataclasses
    cfg = dataclasses.replace(wl.CONFIGS[base], n_q_heads=hq, n_kv_heads=hkv, batch=6,
                              lengths=("uniform", 1, 700), samples_per_prompt=1,
                              min_pool_blocks=0, block_size=bs)
    side = setup_config(cfg, growth=5)
    run_rounds(cfg, side, 3)            # parity of the automatic choice, round by round
    seqs = np.asarray(side.seqs, dtype=np.int64)
    max_blocks = max(len(side.orc.bm.tables[s]) for s in side.seqs) + 2
    step = pk.Step(side.pool, len(seqs), max_blocks, cfg.n_q_heads, cfg.q_dtype)
    out = torch.empty((len(seqs), hq, cfg.head_dim), device="cuda",
                      dtype=torch.bfloat16 if cfg.q_dtype == "bf16" else torch.float16)
    q, kn, vn = step_inputs(side, seqs, 3)
    pk.pkv_decode_step(step, seqs, to_torch(q, cfg.q_dtype), to_torch(kn, cfg.q_dtype),
                       to_torch(vn, cfg.q_dtype), cfg.scale, out)
    torch.cuda.synchronize()
    assert step.last_kernel == expect


def test_step_runtime_rejects_table_overflow_without_changes():
    cfg = wl.CONFIGS["toy"]
    side = setup_config(cfg)
    seqs = np.asarray(side.seqs, dtype=np.int64)
    step = pk.Step(side.pool, len(seqs), 1, 1, "f32")     # max_blocks 1: too small
    before = pk.bt_stats(side.pool)
    q = torch.zeros((len(seqs), 1, 32), device="cuda")
    kv = torch.zeros((len(seqs), 1, 32), device="cuda")
    with pytest.raises(pk.PagedKVError) as e:
        pk.pkv_decode_step(step, seqs, q, kv, kv, 0.1, q.clone())
    assert e.value.status == pk.PKV_ERR_INVALID_ARG
    assert pk.bt_stats(side.pool) == before


@pytest.mark.parametrize("lengths,batch", [(("uniform", 1, 60), 6), (("uniform", 1800, 2000), 10)])
def test_step_runtime_reordered_batches(lengths, batch):
    # the device keeps the tables between rounds and receives only changed
    # entries; reordering the batch (or switching to other sequences) must
    # re-send whole rows - through the parameter block when they fit, through
    # the packed upload when they do not
    import dataclasses
    cfg = dataclasses.replace(wl.CONFIGS["opt13b"], n_q_heads=2, n_kv_heads=2, batch=batch,
                              lengths=lengths, min_pool_blocks=0)
    side = setup_config(cfg, growth=6)
    ids = np.asarray(side.seqs, dtype=np.int64)
    orders = [ids, ids, ids[::-1].copy(), ids[::-1].copy(), ids[: batch // 2], ids]
    max_blocks = max(len(side.orc.bm.tables[s]) for s in side.seqs) + 2
    step = pk.Step(side.pool, batch, max_blocks, 2, "f16")
    out = torch.empty((batch, 2, 128), device="cuda", dtype=torch.float16)
    for t, seqs in enumerate(orders):
        q, kn, vn = step_inputs(side, seqs, t)
        o = out[: len(seqs)]
        pk.pkv_decode_step(step, seqs, to_torch(q, "f16"), to_torch(kn, "f16"), to_torch(vn, "f16"),
                           cfg.scale, o)
        side.orc.append(list(seqs), kn, vn, "f16")
        ref = side.orc.attend(list(seqs), q, "f16", cfg.scale)
        torch.cuda.synchronize()
        compare_out(to_f64(from_torch(o, "f16"), "f16"), ref, "f16")
    check_pool_bytes(side)
    assert pk.pkv_device_error(side.pool) == 0


def test_step_runtime_evicts_rows_of_sequences_not_in_the_batch():
    # two disjoint batches alternate through a runtime that keeps device rows
    # for only one batch's worth of sequences: every switch evicts rows and
    # sends whole tables again
    import dataclasses
    cfg = dataclasses.replace(wl.CONFIGS["opt13b"], n_q_heads=2, n_kv_heads=2, batch=8,
                              lengths=("uniform", 20, 300), min_pool_blocks=0)
    side = setup_config(cfg, growth=8)
    a = np.arange(0, 4, dtype=np.int64)
    b = np.arange(4, 8, dtype=np.int64)
    step = pk.Step(side.pool, 4, 32, 2, "f16", max_seqs=4)
    out = torch.empty((4, 2, 128), device="cuda", dtype=torch.float16)
    for t, seqs in enumerate([a, b, a, a, b, a, b, b]):
        q, kn, vn = step_inputs(side, seqs, t)
        pk.pkv_decode_step(step, seqs, to_torch(q, "f16"), to_torch(kn, "f16"), to_torch(vn, "f16"),
                           cfg.scale, out)
        side.orc.append(list(seqs), kn, vn, "f16")
        ref = side.orc.attend(list(seqs), q, "f16", cfg.scale)
        torch.cuda.synchronize()
        compare_out(to_f64(from_torch(out, "f16"), "f16"), ref, "f16")
    assert pk.pkv_device_error(side.pool) == 0


@pytest.mark.parametrize("dt,bs", [("f16", 16), ("bf16", 4), ("fp8", 16), ("f32", 1)])
def test_swap_out_and_in(dt, bs):
    # "KV 缓存与分页注意力" section 放不下的时候: a sequence gives up all of its blocks
    # to CPU memory and comes back later; its attention afterwards equals the
    # oracle's, the host copy holds exactly its stored rows, and its new
    # blocks follow the free queue like any admission
    import dataclasses
    base = "fp8" if dt == "fp8" else "opt13b"
    cfg = dataclasses.replace(wl.CONFIGS[base], n_q_heads=4, n_kv_heads=2, head_dim=64 if dt != "fp8" else 128,
                              kv_dtype=dt, q_dtype="f16" if dt == "fp8" else dt, block_size=bs,
                              batch=5, lengths=("uniform", 30, 200), min_pool_blocks=0)
    side = setup_config(cfg, growth=4)
    seqs = list(range(cfg.batch))
    from paged_harness import decode_step
    decode_step(side, seqs, 0)
    victim = 2
    bb = pk.block_bytes(side.pool)
    nb = len(side.orc.bm.tables[victim])
    hk = torch.empty(nb * bb, dtype=torch.uint8).pin_memory()
    hv = torch.empty(nb * bb, dtype=torch.uint8).pin_memory()
    n_blocks, n_tokens = pk.kv_swap_out(side.pool, victim, hk, hv)
    torch.cuda.synchronize()
    krows, vrows = side.orc.swap_out(victim)
    assert (n_blocks, n_tokens) == (nb, len(krows))
    store = {"f32": np.float32, "f16": np.float16, "bf16": np.uint16, "fp8": np.uint8}[dt]
    img_k = hk.numpy().view(store).reshape(nb, cfg.n_kv_heads, bs, cfg.head_dim)
    got = np.stack([img_k[t // bs, :, t % bs, :] for t in range(n_tokens)])
    assert np.array_equal(got.view(np.uint8), krows.view(np.uint8))
    # the freed blocks are reused by the other sequences' next rounds
    others = [s for s in seqs if s != victim]
    decode_step(side, others, 1)
    with pytest.raises(pk.PagedKVError):
        pk.kv_swap_in(side.pool, victim, hk[:bb], hv[:bb], n_tokens)        # buffer too small
    pk.kv_swap_in(side.pool, victim, hk, hv, n_tokens)
    assert side.orc.swap_in(victim, krows, vrows) is not None
    tables, _, _ = pk.bt_export(side.pool, [victim], nb)
    assert tables[0].tolist() == side.orc.bm.tables[victim]
    side.seqs = sorted(side.orc.bm.tables)
    gpu, ref, _ = decode_step(side, seqs, 2)
    compare_out(gpu, ref, "fp8" if dt == "fp8" else dt)
    check_pool_bytes(side)


@pytest.mark.parametrize("bs", [4, 16])
def test_prefix_cached_prompts(bs):
    # "KV 缓存与分页注意力" section 后来的做法: prompts that start with the same tokens
    # share the registered blocks; the rows of a token depend on its prefix
    # (as a model's would), so the shared blocks hold exactly the rows each
    # sharer would have written; only the uncached tail is appended
    import dataclasses
    import zlib
    cfg = dataclasses.replace(wl.CONFIGS["opt13b"], n_q_heads=2, n_kv_heads=2, block_size=bs,
                              batch=4, lengths=("fixed", 0), min_pool_blocks=0)
    from paged_harness import make_pair, decode_step
    side = make_pair(cfg, 128, np.random.default_rng(3).permutation(128).astype(np.int32))
    pk.bt_set_prefix_caching(side.pool, True)
    side.orc.bm.set_prefix_caching(True)
    rnd = np.random.default_rng(5)
    system = rnd.integers(0, 50, size=4 * bs + 3).tolist()
    prompts = [system + rnd.integers(0, 50, size=5).tolist(),
               system[: 4 * bs] + rnd.integers(0, 50, size=7).tolist(),
               system[: 2 * bs + 1] + rnd.integers(0, 50, size=2 * bs).tolist(),
               rnd.integers(0, 50, size=3 * bs).tolist()]

    def rows(tokens):
        out_k, out_v = [], []
        for j in range(len(tokens)):
            key = zlib.crc32(np.asarray(tokens[: j + 1], np.int32).tobytes())
            g = np.random.default_rng([11, key])
            out_k.append(g.standard_normal((2, 128), dtype=np.float32))
            out_v.append(g.standard_normal((2, 128), dtype=np.float32))
        return wl.round_to(np.stack(out_k), "f16"), wl.round_to(np.stack(out_v), "f16")

    cached = []
    for s, toks in enumerate(prompts):
        k, v = rows(toks)
        slots, n_cached = pk.bt_alloc_prefix(side.pool, s, toks)
        o_slots, o_cached = side.orc.admit_prefix(s, toks, k, v, "f16")
        assert slots.tolist() == o_slots and n_cached == o_cached
        cached.append(n_cached)
        if n_cached < len(toks):
            pk.kv_append(side.pool, torch.from_numpy(slots[n_cached:].copy()).cuda(),
                         to_torch(k[n_cached:], "f16"), to_torch(v[n_cached:], "f16"))
        side.seqs.append(s)
    assert cached == [0, 4 * bs, 2 * bs, 0]
    assert pk.bt_stats(side.pool)["prefix_hit_tokens"] == 6 * bs
    gpu, ref, _ = decode_step(side, [0, 1, 2, 3], 0)
    compare_out(gpu, ref, "f16")
    check_pool_bytes(side)


@pytest.mark.parametrize("base,dt,pinned,packed", [("opt13b", "f16", True, False),
                                                   ("llama2_70b", "bf16", False, False),
                                                   ("fp8_gqa", "f16", True, True),
                                                   ("opt13b", "f16", False, True)])
def test_step_runtime_host_buffers(base, dt, pinned, packed):
    # the host-buffer entry point: q/k/v in from host memory, out back to it,
    # round after round against the oracle
    import dataclasses
    cfg = dataclasses.replace(wl.CONFIGS[base], n_q_heads=8, n_kv_heads=2 if base != "opt13b" else 8,
                              batch=7, lengths=("uniform", 1, 900), min_pool_blocks=0)
    side = setup_config(cfg, growth=4)
    seqs = np.asarray(side.seqs, dtype=np.int64)
    max_blocks = max(len(side.orc.bm.tables[s]) for s in side.seqs) + 2
    step = pk.Step(side.pool, len(seqs), max_blocks, cfg.n_q_heads, cfg.q_dtype)
    tdt = torch.bfloat16 if cfg.q_dtype == "bf16" else torch.float16
    out = torch.empty((len(seqs), cfg.n_q_heads, cfg.head_dim), dtype=tdt)
    if pinned:
        out = out.pin_memory()
    for t in range(4):
        q, kn, vn = step_inputs(side, seqs, t)
        hq, hk, hv = (to_torch(a, cfg.q_dtype).cpu() for a in (q, kn, vn))
        if packed:   # one host buffer q | k | v: the inputs travel in one copy
            buf = torch.cat([hq.flatten(), hk.flatten(), hv.flatten()])
            buf = buf.pin_memory() if pinned else buf
            nq, nk = hq.numel(), hk.numel()
            hq, hk, hv = buf[:nq].view(hq.shape), buf[nq:nq + nk].view(hk.shape), buf[nq + nk:].view(hv.shape)
        elif pinned:
            hq, hk, hv = hq.pin_memory(), hk.pin_memory(), hv.pin_memory()
        pk.pkv_decode_step_host(step, seqs, hq, hk, hv, cfg.scale, out)
        side.orc.append(list(seqs), kn, vn, cfg.q_dtype)
        ref = side.orc.attend(list(seqs), q, cfg.q_dtype, cfg.scale)
        gpu = to_f64(from_torch(out, cfg.q_dtype), cfg.q_dtype)   # no synchronize: the call waited
        compare_out(gpu, ref, "fp8" if cfg.kv_dtype == "fp8" else cfg.q_dtype)
    assert pk.pkv_device_error(side.pool) == 0
    # a rejected batch (table overflow) changes nothing and reports INVALID_ARG
    small = pk.Step(side.pool, len(seqs), 1, cfg.n_q_heads, cfg.q_dtype)
    with pytest.raises(pk.PagedKVError):
        pk.pkv_decode_step_host(small, seqs, hq, hk, hv, cfg.scale, out)
