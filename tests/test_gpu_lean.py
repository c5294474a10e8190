"""GPU parity of the stage-balanced tensor-core decode (persistent workers that
share the batch's 16-token stages equally, split pairs merged by a second launch)
against the CPU oracle: block sizes, head groupings, ragged and degenerate
batches, pairs split over many CTAs, invalid lengths and block ids, and the
decode-step runtime over many rounds."""

import dataclasses

import numpy as np
import pytest
import torch

import pagedattention_decode_02_b200 as pk
import workloads as wl
from paged_harness import (compare_out, decode_step, from_torch, setup_config, step_inputs,
                           to_torch)
from oracle.numerics import to_f64

pytestmark = pytest.mark.gpu

LEAN = pk.PKV_KERNEL_LEAN


def small(base: str, **kw) -> wl.Config:
    return dataclasses.replace(wl.CONFIGS[base], **kw)


CASES = [
    (dt, d, bs, hq, hkv)
    for dt in ("f16", "bf16")
    for d in (64, 128)
    for bs in (1, 4, 16, 64)
    for (hq, hkv) in ((3, 3), (4, 2), (64, 8), (71, 1), (128, 1))
    if not (bs == 1 and hq >= 64)
] + [("bf16", 128, bs, 16, 2) for bs in (2, 8, 32)]


@pytest.mark.parametrize("dt,d,bs,hq,hkv", CASES)
def test_lean_small(dt, d, bs, hq, hkv):
    cfg = small("llama2_70b", n_q_heads=hq, n_kv_heads=hkv, head_dim=d, kv_dtype=dt, q_dtype=dt,
                block_size=bs, batch=5, lengths=("uniform", 1, 300))
    side = setup_config(cfg, seed=bs + hq + d)
    gpu, ref, _ = decode_step(side, list(range(cfg.batch)), 0, kernel=LEAN)
    compare_out(gpu, ref, dt)


@pytest.mark.parametrize("hq,hkv,d", [(8, 1, 128), (64, 8, 128), (1, 1, 64)])
def test_lean_one_long_sequence(hq, hkv, d):
    # one pair cut into pieces over hundreds of CTAs, merged by the last one
    cfg = small("llama2_70b", n_q_heads=hq, n_kv_heads=hkv, head_dim=d, block_size=16, batch=2,
                lengths=("fixed", 6000))
    side = setup_config(cfg, seed=5)
    gpu, ref, info = decode_step(side, [0, 1], 0, kernel=LEAN)
    assert int(info["lens"].min()) == 6001
    compare_out(gpu, ref, "bf16")


def test_lean_many_short_sequences():
    # many pairs per CTA share, lengths 1..20 (one or two stages each)
    cfg = small("llama2_70b", n_q_heads=16, n_kv_heads=4, head_dim=128, block_size=16, batch=300,
                lengths=("uniform", 0, 20))
    side = setup_config(cfg, seed=9)
    gpu, ref, _ = decode_step(side, list(range(cfg.batch)), 0, kernel=LEAN)
    compare_out(gpu, ref, "bf16")


def test_lean_mixed_lengths_auto_choice():
    # the automatic choice and the stage-balanced kernel, round after round
    cfg = small("llama2_70b", n_q_heads=32, n_kv_heads=4, head_dim=128, block_size=16, batch=40,
                lengths=("loguniform", 1, 3000))
    side = setup_config(cfg, seed=13, growth=2)
    for step, kernel in ((0, pk.PKV_KERNEL_AUTO), (1, LEAN)):
        gpu, ref, _ = decode_step(side, list(range(cfg.batch)), step, kernel=kernel)
        compare_out(gpu, ref, "bf16")


def test_lean_invalid_length_and_block_id():
    pool = pk.kv_pool_create(16, 16, 2, 128, "bf16")
    kb, vb = pool.device_buffers()
    for buf in (kb, vb):
        vals = torch.randn(buf.numel() // 2, device="cuda", dtype=torch.bfloat16)
        buf.copy_(vals.view(torch.uint8).view(buf.shape))
    q = torch.randn(3, 8, 128, device="cuda", dtype=torch.bfloat16)
    tables = torch.tensor([[0, 1, 2], [3, 4, 5], [6, 7, 8]], dtype=torch.int32, device="cuda")
    lens = torch.tensor([0, 40, 49], dtype=torch.int32, device="cuda")   # 49 > 3 blocks * 16
    out = pk.paged_decode_attention(pool, q, tables, lens, 0.1, kernel=LEAN)
    bits = pk.pkv_device_error(pool)
    assert bits & pk.PKV_DEVERR_CONTEXT_LEN
    assert torch.all(out[0] == 0) and torch.all(out[2] == 0)
    assert torch.all(torch.isfinite(out[1].float()))
    # an out-of-range block id: its piece contributes nothing, the error bit is set
    tables = torch.tensor([[0, 99, 2], [3, 4, 5], [6, -1, 8]], dtype=torch.int32, device="cuda")
    lens = torch.tensor([20, 40, 10], dtype=torch.int32, device="cuda")
    out = pk.paged_decode_attention(pool, q, tables, lens, 0.1, kernel=LEAN)
    assert pk.pkv_device_error(pool) & pk.PKV_DEVERR_BLOCK_ID
    assert torch.all(torch.isfinite(out.float()))
    assert pk.pkv_device_error(pool) == 0


def test_lean_refuses_unsupported():
    pool = pk.kv_pool_create(16, 16, 1, 64, "f32")
    q = torch.zeros(1, 4, 64, device="cuda", dtype=torch.float32)
    tables = torch.zeros(1, 2, dtype=torch.int32, device="cuda")
    lens = torch.ones(1, dtype=torch.int32, device="cuda")
    with pytest.raises(pk.PagedKVError):
        pk.paged_decode_attention(pool, q, tables, lens, 0.1, kernel=LEAN)
    pool = pk.kv_pool_create(16, 16, 1, 64, "f16")
    q = torch.zeros(1, 4, 64, device="cuda", dtype=torch.float16)
    with pytest.raises(pk.PagedKVError):     # no workspace
        st = pk._lib.paged_decode_attention_ex(pool.handle, q.data_ptr(), pk.PKV_F16,
                                               tables.data_ptr(), 2, lens.data_ptr(), 1, 4, 0.1,
                                               q.data_ptr(), None, 0, 0, LEAN, None)
        pk._check(st, "ex")


@pytest.mark.parametrize("hq,hkv", [(64, 8), (71, 1)])
def test_lean_step_runtime_many_rounds(hq, hkv):
    # every round of a multi-round run must merge its split pairs correctly
    d = 128 if hkv == 8 else 64
    dt = "bf16" if hkv == 8 else "f16"
    cfg = small("llama2_70b", n_q_heads=hq, n_kv_heads=hkv, head_dim=d, kv_dtype=dt, q_dtype=dt,
                block_size=16, batch=12, lengths=("loguniform", 16, 2500))
    side = setup_config(cfg, seed=21, growth=6)
    seqs = np.asarray(side.seqs, dtype=np.int64)
    max_blocks = max(len(side.orc.bm.tables[s]) for s in side.seqs) + 2
    step = pk.Step(side.pool, len(seqs), max_blocks, hq, dt)
    out = torch.empty((len(seqs), hq, d), device="cuda",
                      dtype=torch.bfloat16 if dt == "bf16" else torch.float16)
    for r in range(6):
        q, kn, vn = step_inputs(side, seqs, r)
        pk.pkv_decode_step(step, seqs, to_torch(q, dt), to_torch(kn, dt), to_torch(vn, dt),
                           cfg.scale, out)
        if r > 0:                               # tables already resident
            assert step.last_launches == 2      # prologue + decode (merge included)
        side.orc.append(list(seqs), kn, vn, dt)
        ref = side.orc.attend(list(seqs), q, dt, cfg.scale)
        torch.cuda.synchronize()
        compare_out(to_f64(from_torch(out, dt), dt), ref, dt)
    assert pk.pkv_device_error(side.pool) == 0
