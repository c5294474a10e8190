"""GPU parity: the CUDA decode step (block tables, copy-on-write, append,
paged decode attention, split-context merge) against the CPU oracle.

Block tables, slots, copy pairs and pool bytes are compared bit-exactly;
attention outputs within the stated tolerances (fp32 1e-5, fp16 3e-3, bf16
1.5e-2, FP8 1.5e-2 after dequantisation), max abs over every compared element.
"""

import dataclasses
import numpy as np
import pytest
import torch

import pagedattention_decode_02_b200 as pk
import workloads as wl
from paged_harness import (TOL, check_pool_bytes, compare_out, decode_step, from_torch,
                           make_pair, admit, setup_config, to_torch)
from oracle.numerics import to_f64

pytestmark = pytest.mark.gpu


def small(base: str, **kw) -> wl.Config:
    return dataclasses.replace(wl.CONFIGS[base], **kw)


# ---------------------------------------------------------------------------
# config 1: the exhibit's toy pool, full oracle
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("partition", [0, -1, 16])
def test_toy_config_full(partition):
    cfg = wl.CONFIGS["toy"]
    side = setup_config(cfg)
    assert side.pool.num_blocks == 44
    gpu, ref, info = decode_step(side, list(range(cfg.batch)), 0, partition_tokens=partition)
    compare_out(gpu, ref, "f32")
    check_pool_bytes(side)
    # blocks handed out in arrival order from an identity free queue
    first = info["tables"][0][info["tables"][0] >= 0]
    assert first.tolist() == list(range(len(first)))


# ---------------------------------------------------------------------------
# small MHA / GQA cases spanning several stages and a ragged tail
# ---------------------------------------------------------------------------
MHA_CASES = [
    (dt, d, bs, part)
    for dt in ("f32", "f16", "bf16")
    for d in (32, 64, 128)
    for bs in (1, 4, 16, 64)
    for part in (0, -1, 16, 48)
    if not (dt == "f32" and d == 128 and bs == 1)
]


@pytest.mark.parametrize("dt,d,bs,part", MHA_CASES)
@pytest.mark.parametrize("kernel", [pk.PKV_KERNEL_SIMT_BULK, pk.PKV_KERNEL_SIMT])
def test_mha_small(dt, d, bs, part, kernel):
    cfg = small("opt13b", n_q_heads=3, n_kv_heads=3, head_dim=d, kv_dtype=dt, q_dtype=dt,
                block_size=bs, batch=5, lengths=("uniform", 1, 150), min_pool_blocks=0)
    side = setup_config(cfg, seed=d + bs)
    gpu, ref, _ = decode_step(side, list(range(cfg.batch)), 0, partition_tokens=part, kernel=kernel)
    compare_out(gpu, ref, dt)
    check_pool_bytes(side)


@pytest.mark.parametrize("dt,d", [("f32", 32), ("f32", 64), ("f32", 128), ("f16", 64), ("f16", 128),
                                  ("bf16", 64), ("bf16", 128)])
@pytest.mark.parametrize("bs", [1, 2, 8, 16, 32])
def test_simt_tma_small(dt, d, bs):
    # the swizzled-TMA CUDA-core kernel, forced, with grouped heads too
    cfg = small("opt13b", n_q_heads=6, n_kv_heads=3, head_dim=d, kv_dtype=dt, q_dtype=dt,
                block_size=bs, batch=5, lengths=("uniform", 1, 300), min_pool_blocks=0)
    side = setup_config(cfg, seed=3 * d + bs, growth=3)
    for part in (0, 16, 64):
        gpu, ref, _ = decode_step(side, list(range(cfg.batch)), part // 16,
                                  partition_tokens=part, kernel=pk.PKV_KERNEL_SIMT_TMA)
        compare_out(gpu, ref, dt)


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("hq,hkv", [(4, 2), (8, 1), (16, 2), (12, 4)])
@pytest.mark.parametrize("kernel", [pk.PKV_KERNEL_SIMT, pk.PKV_KERNEL_AUTO])
@pytest.mark.parametrize("part", [0, 32])
def test_gqa_small(dt, hq, hkv, kernel, part):
    cfg = small("llama2_70b", n_q_heads=hq, n_kv_heads=hkv, head_dim=64, kv_dtype=dt, q_dtype=dt,
                block_size=16, batch=4, lengths=("uniform", 1, 200))
    side = setup_config(cfg, seed=hq * 7 + hkv)
    gpu, ref, _ = decode_step(side, list(range(cfg.batch)), 0, partition_tokens=part, kernel=kernel)
    compare_out(gpu, ref, dt)


@pytest.mark.parametrize("bs", [1, 2, 4, 8, 16, 32, 64])
@pytest.mark.parametrize("qdt", ["f16", "bf16"])
@pytest.mark.parametrize("kernel", [pk.PKV_KERNEL_SIMT_BULK, pk.PKV_KERNEL_AUTO])
def test_fp8_small(bs, qdt, kernel):
    cfg = small("fp8", n_q_heads=4, n_kv_heads=4, q_dtype=qdt, block_size=bs, batch=6,
                lengths=("uniform", 1, 130))
    side = setup_config(cfg, seed=bs)
    gpu, ref, _ = decode_step(side, list(range(cfg.batch)), 0, kernel=kernel)
    compare_out(gpu, ref, "fp8")
    check_pool_bytes(side)


@pytest.mark.parametrize("bs", [1, 2, 4, 8, 16, 64])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 4), (16, 2), (8, 1), (5, 1)])
@pytest.mark.parametrize("part", [0, 32])
def test_fp8_tensor_small(bs, hq, hkv, part):
    # FP8 codes converted to f16 in registers feed the tensor-core stage math
    cfg = small("fp8", n_q_heads=hq, n_kv_heads=hkv, block_size=bs, batch=5,
                lengths=("uniform", 1, 300))
    side = setup_config(cfg, seed=bs * 3 + hq)
    gpu, ref, _ = decode_step(side, list(range(cfg.batch)), 0, partition_tokens=part,
                              kernel=pk.PKV_KERNEL_TENSOR)
    compare_out(gpu, ref, "fp8")


def test_fp8_tensor_refusals():
    # bf16 queries, head_dim 64 and more than 8 heads per KV head stay on the CUDA cores
    tables = torch.zeros(1, 2, dtype=torch.int32, device="cuda")
    lens = torch.ones(1, dtype=torch.int32, device="cuda")
    for d, hq, qdt in ((128, 4, torch.bfloat16), (64, 4, torch.float16), (128, 16, torch.float16)):
        pool = pk.kv_pool_create(8, 16, 1, d, "fp8")
        for buf in pool.device_buffers():
            buf.zero_()
        q = torch.zeros(1, hq, d, device="cuda", dtype=qdt)
        with pytest.raises(pk.PagedKVError):
            pk.paged_decode_attention(pool, q, tables, lens, 0.1, kernel=pk.PKV_KERNEL_TENSOR)
        out = pk.paged_decode_attention(pool, q, tables, lens, 0.1)   # the automatic choice runs
        assert torch.all(torch.isfinite(out.float()))


# ---------------------------------------------------------------------------
# edge cases
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_single_token_returns_its_value(dt):
    cfg = small("opt13b", n_q_heads=2, n_kv_heads=2, head_dim=64, kv_dtype=dt, q_dtype=dt,
                block_size=16, batch=3, lengths=("fixed", 0))
    side = make_pair(cfg, 8, np.arange(8, dtype=np.int32))
    admit(side, [0, 1, 2], [0, 0, 0])
    gpu, ref, _ = decode_step(side, [0, 1, 2], 0)
    compare_out(gpu, ref, dt)
    kh, vh = side.orc.history(1)
    assert np.array_equal(gpu[1], to_f64(vh[0], dt))    # out = v exactly


def test_contexts_on_block_boundaries():
    cfg = small("opt13b", n_q_heads=2, n_kv_heads=2, head_dim=128, block_size=16, batch=4,
                lengths=("fixed", 0))
    side = make_pair(cfg, 64, np.arange(64, dtype=np.int32)[::-1].copy())
    admit(side, [0, 1, 2, 3], [15, 31, 63, 127])        # +1 on append -> multiples of 16
    gpu, ref, info = decode_step(side, [0, 1, 2, 3], 0)
    assert info["lens"].tolist() == [16, 32, 64, 128]
    compare_out(gpu, ref, "f16")
    gpu, ref, _ = decode_step(side, [0, 1, 2, 3], 1)     # next append opens a fresh block
    compare_out(gpu, ref, "f16")


def test_bad_context_len_and_block_id_set_error_bits():
    cfg = small("opt13b", n_q_heads=2, n_kv_heads=2, head_dim=64, block_size=4, batch=2,
                lengths=("fixed", 0))
    pool = pk.kv_pool_create(8, 4, 2, 64, "f16")
    q = torch.randn(2, 2, 64, device="cuda", dtype=torch.float16)
    tables = torch.tensor([[0, 1], [2, 3]], dtype=torch.int32, device="cuda")
    lens = torch.tensor([0, 5], dtype=torch.int32, device="cuda")
    out = pk.paged_decode_attention(pool, q, tables, lens, 0.125)
    bits = pk.pkv_device_error(pool)
    assert bits & pk.PKV_DEVERR_CONTEXT_LEN
    assert torch.all(out[0] == 0)
    lens = torch.tensor([3, 9], dtype=torch.int32, device="cuda")     # 9 > 2 blocks * 4
    pk.paged_decode_attention(pool, q, tables, lens, 0.125)
    assert pk.pkv_device_error(pool) & pk.PKV_DEVERR_CONTEXT_LEN
    tables = torch.tensor([[0, 99], [2, -1]], dtype=torch.int32, device="cuda")
    lens = torch.tensor([6, 2], dtype=torch.int32, device="cuda")
    pk.paged_decode_attention(pool, q, tables, lens, 0.125)
    assert pk.pkv_device_error(pool) & pk.PKV_DEVERR_BLOCK_ID
    assert pk.pkv_device_error(pool) == 0                               # cleared
    # slot out of range on append
    slots = torch.tensor([0, 10 ** 6], dtype=torch.int32, device="cuda")
    kv = torch.randn(2, 2, 64, device="cuda", dtype=torch.float16)
    pk.kv_append(pool, slots, kv, kv)
    assert pk.pkv_device_error(pool) & pk.PKV_DEVERR_SLOT


def test_host_side_argument_errors():
    pool = pk.kv_pool_create(8, 4, 2, 64, "f16")
    q = torch.randn(2, 3, 64, device="cuda", dtype=torch.float16)   # 3 % 2 != 0
    tables = torch.zeros(2, 2, dtype=torch.int32, device="cuda")
    lens = torch.ones(2, dtype=torch.int32, device="cuda")
    with pytest.raises(pk.PagedKVError):
        pk.paged_decode_attention(pool, q, tables, lens, 0.1)
    q = torch.randn(2, 2, 64, device="cuda", dtype=torch.bfloat16)  # wrong dtype
    with pytest.raises(pk.PagedKVError):
        pk.paged_decode_attention(pool, q, tables, lens, 0.1)
    q = torch.randn(2, 2, 64, device="cuda", dtype=torch.float16)
    tables8 = torch.zeros(2, 8, dtype=torch.int32, device="cuda")  # 32 tokens: 2 partitions of 16
    with pytest.raises(pk.PagedKVError):                               # split without workspace
        st = pk._lib.paged_decode_attention_ex(pool.handle, q.data_ptr(), pk.PKV_F16,
                                               tables8.data_ptr(), 8, lens.data_ptr(), 2, 2, 0.1,
                                               q.data_ptr(), None, 0, 16, 0, None)
        pk._check(st, "ex")
    with pytest.raises(pk.PagedKVError):                               # tensor path, G == 1
        pk.paged_decode_attention(pool, q, tables, lens, 0.1, kernel=pk.PKV_KERNEL_TENSOR)


def test_block_copy_whole_blocks_bit_exact():
    pool = pk.kv_pool_create(6, 4, 3, 64, "bf16")
    kb, vb = pool.device_buffers()
    kb.copy_(torch.randint(0, 256, kb.shape, dtype=torch.uint8, device="cuda"))
    vb.copy_(torch.randint(0, 256, vb.shape, dtype=torch.uint8, device="cuda"))
    k0, v0 = kb.clone(), vb.clone()
    src = torch.tensor([0, 2], dtype=torch.int32, device="cuda")
    dst = torch.tensor([5, 3], dtype=torch.int32, device="cuda")
    pk.block_copy(pool, src, dst)
    torch.cuda.synchronize()
    assert torch.equal(kb[5], k0[0]) and torch.equal(kb[3], k0[2])
    assert torch.equal(vb[5], v0[0]) and torch.equal(vb[3], v0[2])
    for b in (0, 1, 2, 4):
        assert torch.equal(kb[b], k0[b]) and torch.equal(vb[b], v0[b])


def test_caller_owned_buffers():
    cfg = small("opt13b", n_q_heads=2, n_kv_heads=2, head_dim=128, block_size=16, batch=3,
                lengths=("uniform", 10, 90))
    side = setup_config(cfg, torch_buffers=True)
    gpu, ref, _ = decode_step(side, list(range(3)), 0)
    compare_out(gpu, ref, "f16")
    check_pool_bytes(side)


# ---------------------------------------------------------------------------
# full-size workloads through the public call (automatic partitioning and
# kernel choice); every head of every sequence is compared
# ---------------------------------------------------------------------------


@pytest.mark.slow
@pytest.mark.parametrize("partition", [0, 512])   # automatic (unsplit: 1,200 CTAs fill the GPU), split
def test_opt13b_full(partition):
    cfg = wl.CONFIGS["opt13b"]
    side = setup_config(cfg)
    gpu, ref, info = decode_step(side, list(range(cfg.batch)), 0, partition_tokens=partition)
    compare_out(gpu, ref, "f16")
    check_pool_bytes(side)
    assert side.pool.num_blocks == max(982, wl.pool_blocks(cfg, wl.history_lengths(cfg, 0), 1))


@pytest.mark.slow
def test_llama2_70b_full():
    cfg = wl.CONFIGS["llama2_70b"]
    side = setup_config(cfg)
    gpu, ref, info = decode_step(side, list(range(cfg.batch)), 0)
    compare_out(gpu, ref, "bf16")
    assert int(info["lens"].max()) > 512          # the split path ran


@pytest.mark.slow
@pytest.mark.parametrize("variant", ["a", "b"])
def test_falcon7b_sharing_all_steps(variant):
    cfg = wl.CONFIGS["falcon7b"]
    side = setup_config(cfg, variant=variant, growth=cfg.steps)
    seqs = list(range(cfg.batch))
    total_pairs = 0
    for step in range(cfg.steps):
        gpu, ref, info = decode_step(side, seqs, step)
        compare_out(gpu, ref, "f16")
        total_pairs += len(info["pairs"])
        if step in (0, 1, cfg.steps - 1):
            check_pool_bytes(side)
    st = pk.bt_stats(side.pool)
    if variant == "a":
        # 512 = 32 x 16: the prompts' last blocks are full, nothing is copied
        assert total_pairs == 0 and st["cow_count"] == 0
    else:
        # every prompt's partial last block: 3 of its 4 samples copy
        assert total_pairs == 16 * 3 and st["cow_count"] == 16 * 3
    # prompt blocks stay shared by all four samples
    t0 = side.orc.bm.tables[0]
    assert pk.bt_refcount(side.pool, t0[0]) == 4


@pytest.mark.slow
@pytest.mark.parametrize("kernel", [pk.PKV_KERNEL_AUTO, pk.PKV_KERNEL_TENSOR, pk.PKV_KERNEL_SIMT])
def test_fp8_gqa_full(kernel):
    # the Llama-2-70B-shaped batch on an FP8 pool (f16 q/out), every head
    cfg = wl.CONFIGS["fp8_gqa"]
    side = setup_config(cfg)
    seqs = list(range(cfg.batch))
    gpu, ref, _ = decode_step(side, seqs, 0, kernel=kernel)
    compare_out(gpu, ref, "fp8")


@pytest.mark.slow
@pytest.mark.parametrize("bs", [1, 4, 16])   # 4 and 16: the bench's FP8 sub-records
def test_fp8_full(bs):
    cfg = wl.CONFIGS["fp8"].with_block_size(bs)
    side = setup_config(cfg)
    seqs = list(range(cfg.batch))
    gpu, ref, info = decode_step(side, seqs, 0)
    compare_out(gpu, ref, "fp8")
    check_pool_bytes(side, seqs[:8])


# ---------------------------------------------------------------------------
# tensor-core path for grouped heads, forced
# ---------------------------------------------------------------------------
TC_CASES = [
    (dt, d, bs, hq, hkv, part)
    for dt in ("f16", "bf16")
    for d in (64, 128)
    for bs in (8, 16, 32)
    for (hq, hkv) in ((4, 2), (16, 2), (71, 1), (64, 8), (128, 1))
    for part in (0, 32)
    if not (d == 128 and hq == 128 and bs == 32)
] + [("f16", 64, bs, 8, 1, 0) for bs in (1, 2, 4)] + [("bf16", 128, bs, 16, 2, 32) for bs in (1, 2, 4)]


@pytest.mark.parametrize("dt,d,bs,hq,hkv,part", TC_CASES)
def test_tensor_path(dt, d, bs, hq, hkv, part):
    cfg = small("llama2_70b", n_q_heads=hq, n_kv_heads=hkv, head_dim=d, kv_dtype=dt, q_dtype=dt,
                block_size=bs, batch=3, lengths=("uniform", 1, 180))
    side = setup_config(cfg, seed=bs + hq)
    gpu, ref, _ = decode_step(side, list(range(cfg.batch)), 0, partition_tokens=part,
                              kernel=pk.PKV_KERNEL_TENSOR)
    compare_out(gpu, ref, dt)


def test_tensor_path_refuses_unsupported_shapes():
    for dt, d, bs in (("f32", 64, 16), ("f16", 32, 16), ("f16", 64, 24), ("bf16", 128, 12)):
        pool = pk.kv_pool_create(16, bs, 1, d, dt)
        tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[dt]
        q = torch.zeros(1, 4, d, device="cuda", dtype=tdt)
        tables = torch.zeros(1, 2, dtype=torch.int32, device="cuda")
        lens = torch.ones(1, dtype=torch.int32, device="cuda")
        with pytest.raises(pk.PagedKVError):
            pk.paged_decode_attention(pool, q, tables, lens, 0.1, kernel=pk.PKV_KERNEL_TENSOR)
        # the automatic choice falls back to the CUDA-core kernel
        pk.paged_decode_attention(pool, q, tables, lens, 0.1)
