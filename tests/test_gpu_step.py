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
        # prologue (append) + decode; the split partitions are merged inside
        # the decode kernel
        assert step.last_launches == 2
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
    assert launches[-1] == (3 if kernel == pk.PKV_KERNEL_SIMT_BULK else 2)


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
