"""Bounded waits: every kernel's wait on a copy (or on a tensor-core result)
gives up after the pool's wait budget, reports PKV_DEVERR_TIMEOUT, waits with
the default budget for what it still has in flight, and returns - leaving the
CUDA context usable.  No GPU fault, trap or hang is involved:

* the probe kernel waits on a barrier phase that nothing completes (no
  arrival, no copy) and must give up within its budget;
* every decode and prompt kernel runs a full-size-ish launch with a 1 ns
  budget, which makes waits give up while their copies are still on the way
  (the give-up-and-drain branch); the launch must return with no error bit
  other than TIMEOUT, and when no wait gave up its output must still match
  the oracle;
* the same launch with the default budget afterwards matches the oracle
  (the context and the pool survived).
"""

import dataclasses
import time

import numpy as np
import pytest
import torch

import pagedattention_decode_02_b200 as pk
import workloads as wl
from oracle.numerics import to_f64
from paged_harness import TOL, compare_out, from_torch, setup_config, step_inputs, to_torch

pytestmark = pytest.mark.gpu


def test_probe_gives_up_within_its_budget():
    pool = pk.kv_pool_create(4, 16, 1, 64, "f16")
    pk.pkv_set_wait_budget(pool, 2_000_000)          # 2 ms
    t0 = time.perf_counter()
    pk.pkv_wait_probe(pool)
    bits = pk.pkv_device_error(pool)
    dt = time.perf_counter() - t0
    assert bits == pk.PKV_DEVERR_TIMEOUT
    assert dt < 1.0                                   # gave up after ~2 ms, not 2 s
    # the default budget is restored by 0; the bit was cleared by the read
    pk.pkv_set_wait_budget(pool, 0)
    assert pk.pkv_device_error(pool) == 0


def test_budget_argument_checks():
    pool = pk.kv_pool_create(4, 16, 1, 64, "f16")
    with pytest.raises(pk.PagedKVError):
        pk.pkv_set_wait_budget(pool, 3_000_000_000)   # above the 2 s default


DECODE_KERNELS = [pk.PKV_KERNEL_SIMT_BULK, pk.PKV_KERNEL_SIMT_TMA, pk.PKV_KERNEL_TENSOR,
                  pk.PKV_KERNEL_LEAN]


def _decode_case(kernel):
    # grouped heads for the tensor-core kernels, one head per KV head else;
    # enough sequences and tokens that every CTA waits on many copies
    hq, hkv = (16, 2) if kernel in (pk.PKV_KERNEL_TENSOR, pk.PKV_KERNEL_LEAN) else (8, 8)
    cfg = dataclasses.replace(wl.CONFIGS["llama2_70b"], n_q_heads=hq, n_kv_heads=hkv,
                              kv_dtype="bf16", q_dtype="bf16", batch=24,
                              lengths=("uniform", 200, 1500))
    side = setup_config(cfg, seed=kernel)
    seqs = list(range(cfg.batch))
    q, kn, vn = step_inputs(side, seqs, 0)
    slots, _, _ = pk.bt_append_batch(side.pool, seqs)
    side.orc.append(seqs, kn, vn, cfg.q_dtype)
    pk.kv_append(side.pool, torch.from_numpy(slots).cuda(), to_torch(kn, "bf16"),
                 to_torch(vn, "bf16"))
    max_blocks = max(pk.bt_num_blocks(side.pool, s) for s in seqs)
    tables, lens, _ = pk.bt_export(side.pool, seqs, max_blocks)
    ref = side.orc.attend(seqs, q, "bf16", cfg.scale)
    return cfg, side, to_torch(q, "bf16"), torch.from_numpy(tables).cuda(), \
        torch.from_numpy(lens).cuda(), ref


@pytest.mark.parametrize("kernel", DECODE_KERNELS)
@pytest.mark.parametrize("part", [0, 128])
def test_decode_kernels_give_up_and_recover(kernel, part):
    if kernel == pk.PKV_KERNEL_LEAN and part:
        pytest.skip("the stage-balanced kernel has no partitions")
    cfg, side, qt, tables, lens, ref = _decode_case(kernel)
    pk.pkv_device_error(side.pool)
    gave_up = 0
    for _ in range(3):
        pk.pkv_set_wait_budget(side.pool, 1)
        out = pk.paged_decode_attention(side.pool, qt, tables, lens, cfg.scale,
                                        partition_tokens=part, kernel=kernel)
        bits = pk.pkv_device_error(side.pool)        # returns: the kernel ended
        assert bits & ~pk.PKV_DEVERR_TIMEOUT == 0, hex(bits)
        if bits:
            gave_up += 1
        else:
            compare_out(to_f64(from_torch(out, "bf16"), "bf16"), ref, "bf16")
    pk.pkv_set_wait_budget(side.pool, 0)
    out = pk.paged_decode_attention(side.pool, qt, tables, lens, cfg.scale,
                                    partition_tokens=part, kernel=kernel)
    assert pk.pkv_device_error(side.pool) == 0
    compare_out(to_f64(from_torch(out, "bf16"), "bf16"), ref, "bf16")
    print(f"kernel {kernel} partition {part}: gave up in {gave_up} of 3 short-budget launches")


@pytest.mark.parametrize("kernel", [pk.PKV_PREFILL_TCGEN05, pk.PKV_PREFILL_MMA_SYNC])
def test_prompt_kernels_give_up_and_recover(kernel):
    cfg = dataclasses.replace(wl.CONFIGS["llama2_70b"], n_q_heads=16, n_kv_heads=2,
                              batch=6, lengths=("uniform", 400, 900))
    side = setup_config(cfg, seed=7)
    seqs = side.seqs
    n = [side.orc.bm.lengths[s] for s in seqs]
    qs = [wl.round_to(wl.prompt_queries(cfg, 0, s, int(k)), "bf16") for s, k in zip(seqs, n)]
    starts = torch.from_numpy(np.concatenate([[0], np.cumsum(n)]).astype(np.int32)).cuda()
    max_blocks = max(pk.bt_num_blocks(side.pool, s) for s in seqs)
    tables, lens, _ = pk.bt_export(side.pool, seqs, max_blocks)
    tables, lens = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    qt = to_torch(np.concatenate(qs), "bf16")
    refs = [side.orc.prefill(s, q, "bf16", cfg.scale) for s, q in zip(seqs, qs)]
    off = np.concatenate([[0], np.cumsum(n)])

    def check(out):
        got = to_f64(from_torch(out, "bf16"), "bf16")
        for i, r in enumerate(refs):
            compare_out(got[off[i]:off[i + 1]], r, "bf16")

    gave_up = 0
    for _ in range(3):
        pk.pkv_set_wait_budget(side.pool, 1)
        out = pk.paged_prefill_attention(side.pool, qt, starts, tables, lens, cfg.scale,
                                         kernel=kernel)
        bits = pk.pkv_device_error(side.pool)
        assert bits & ~pk.PKV_DEVERR_TIMEOUT == 0, hex(bits)
        if bits:
            gave_up += 1
        else:
            check(out)
    pk.pkv_set_wait_budget(side.pool, 0)
    out = pk.paged_prefill_attention(side.pool, qt, starts, tables, lens, cfg.scale,
                                     kernel=kernel)
    assert pk.pkv_device_error(side.pool) == 0
    check(out)
    print(f"prompt kernel {kernel}: gave up in {gave_up} of 3 short-budget launches")
