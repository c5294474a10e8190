"""GPU parity of the prompt-phase attention over the paged cache against the
CPU oracle: prompts with and without a cached prefix, grouped heads, block
sizes, ragged prompt lengths spanning several row tiles and key tiles, prompts
admitted through the prefix cache, and invalid inputs - for both kernels (the
tcgen05 kernel with tensor-memory accumulators, which the library runs by
default, and the mma.sync kernel)."""

import dataclasses

import numpy as np
import pytest
import torch

import pagedattention_decode_02_b200 as pk
import workloads as wl
from paged_harness import TOL, compare_out, from_torch, setup_config, to_torch
from oracle.numerics import to_f64

pytestmark = pytest.mark.gpu


def small(base: str, **kw) -> wl.Config:
    return dataclasses.replace(wl.CONFIGS[base], **kw)


KERNELS = [pk.PKV_PREFILL_TCGEN05, pk.PKV_PREFILL_MMA_SYNC]


def run_prefill(side, prompt_lens, seed=0, kernel=0):
    """Prefill the last n_i tokens of every admitted sequence; -> (gpu, ref)
    lists of float64 [n_i][H_q][d]."""
    cfg = side.cfg
    seqs = side.seqs
    qs = [wl.round_to(wl.prompt_queries(cfg, seed, s, int(n)), cfg.q_dtype)
          for s, n in zip(seqs, prompt_lens)]
    starts = np.concatenate([[0], np.cumsum(prompt_lens)]).astype(np.int32)
    q_all = np.concatenate(qs) if starts[-1] else np.zeros((0, cfg.n_q_heads, cfg.head_dim),
                                                            np.float32)
    max_blocks = max(pk.bt_num_blocks(side.pool, s) for s in seqs)
    tables, lens, _ = pk.bt_export(side.pool, seqs, max_blocks)
    out = pk.paged_prefill_attention(side.pool, to_torch(q_all, cfg.q_dtype),
                                     torch.from_numpy(starts).cuda(),
                                     torch.from_numpy(tables).cuda(),
                                     torch.from_numpy(lens).cuda(), cfg.scale, kernel=kernel)
    torch.cuda.synchronize()
    assert pk.pkv_device_error(side.pool) == 0
    gpu = to_f64(from_torch(out, cfg.q_dtype), cfg.q_dtype)
    refs = [side.orc.prefill(s, q, cfg.q_dtype, cfg.scale) if q.shape[0] else None
            for s, q in zip(seqs, qs)]
    return [gpu[starts[i]:starts[i + 1]] for i in range(len(seqs))], refs


CASES = [
    (dt, d, bs, hq, hkv)
    for dt in ("f16", "bf16")
    for d in (64, 128)
    for bs in (1, 4, 16, 32)
    for (hq, hkv) in ((2, 2), (8, 2), (8, 1), (12, 4))
    if not (bs == 1 and hq == 12)
]


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("dt,d,bs,hq,hkv", CASES)
def test_prefill_small(dt, d, bs, hq, hkv, kernel):
    cfg = small("llama2_70b", n_q_heads=hq, n_kv_heads=hkv, head_dim=d, kv_dtype=dt, q_dtype=dt,
                block_size=bs, batch=4, lengths=("uniform", 1, 200))
    side = setup_config(cfg, seed=d + bs + hq)
    hist = [side.orc.bm.lengths[s] for s in side.seqs]
    rng = np.random.default_rng(bs + hq)
    # prompts from a single token to the whole history (no prefix)
    n = [int(h) if i == 0 else int(rng.integers(1, h + 1)) for i, h in enumerate(hist)]
    gpu, ref = run_prefill(side, n, kernel=kernel)
    for g, r in zip(gpu, ref):
        compare_out(g, r, dt)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("bs", [8, 64, 128, 256])
@pytest.mark.parametrize("d", [64, 128])
def test_prefill_block_sizes(bs, d, kernel):
    # one TMA box per block of up to 128 rows (a 256-token block takes two),
    # over histories of several 128-key tiles with ragged ends
    cfg = small("llama2_70b", n_q_heads=8, n_kv_heads=2, head_dim=d, kv_dtype="bf16",
                q_dtype="bf16", block_size=bs, batch=3, lengths=("uniform", 100, 700))
    side = setup_config(cfg, seed=bs + d)
    hist = [side.orc.bm.lengths[s] for s in side.seqs]
    n = [int(h) if i == 0 else max(1, int(h) // 3) for i, h in enumerate(hist)]
    gpu, ref = run_prefill(side, n, kernel=kernel)
    for g, r in zip(gpu, ref):
        compare_out(g, r, "bf16")


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("hq,hkv,d", [(64, 8, 128), (71, 1, 64), (40, 40, 128), (8, 2, 64)])
def test_prefill_long_prompts(hq, hkv, d, kernel):
    # several row tiles per (sequence, KV head) and several key tiles
    dt = "bf16" if d == 128 else "f16"
    cfg = small("llama2_70b", n_q_heads=hq, n_kv_heads=hkv, head_dim=d, kv_dtype=dt, q_dtype=dt,
                block_size=16, batch=3, lengths=("uniform", 300, 700))
    side = setup_config(cfg, seed=hq)
    hist = [side.orc.bm.lengths[s] for s in side.seqs]
    n = [hist[0], hist[1] // 2, 37]
    gpu, ref = run_prefill(side, n, kernel=kernel)
    for g, r in zip(gpu, ref):
        compare_out(g, r, dt)


@pytest.mark.parametrize("kernel", KERNELS)
def test_prefill_zero_length_prompt_writes_nothing(kernel):
    cfg = small("llama2_70b", n_q_heads=4, n_kv_heads=2, head_dim=64, kv_dtype="f16",
                q_dtype="f16", block_size=16, batch=3, lengths=("uniform", 5, 40))
    side = setup_config(cfg, seed=1)
    gpu, ref = run_prefill(side, [3, 0, 5], kernel=kernel)
    assert gpu[1].shape[0] == 0
    compare_out(gpu[0], ref[0], "f16")
    compare_out(gpu[2], ref[2], "f16")


@pytest.mark.parametrize("kernel", KERNELS)
def test_prefill_after_prefix_cache_hit(kernel):
    # the second prompt shares its first two blocks with the first; only its
    # tail is prefilled, attending to the shared cached blocks
    cfg = small("llama2_70b", n_q_heads=8, n_kv_heads=2, head_dim=128, kv_dtype="bf16",
                q_dtype="bf16", block_size=16, batch=2, lengths=("fixed", 0))
    pool = pk.kv_pool_create(16, 16, 2, 128, "bf16")
    pk.bt_set_prefix_caching(pool, True)
    tokens_a = list(range(1, 41))                 # 40 tokens
    tokens_b = tokens_a[:32] + [99, 98, 97]       # same first two blocks, new tail
    k, v = wl.history_kv(cfg, 0, 0, 40)
    k, v = wl.round_to(k, "bf16"), wl.round_to(v, "bf16")
    slots_a, cached_a = pk.bt_alloc_prefix(pool, 0, tokens_a)
    assert cached_a == 0
    pk.kv_append(pool, torch.from_numpy(slots_a).cuda(), to_torch(k, "bf16"), to_torch(v, "bf16"))
    slots_b, cached_b = pk.bt_alloc_prefix(pool, 1, tokens_b)
    assert cached_b == 32
    kb, vb = wl.history_kv(cfg, 0, 1, 3)
    kb, vb = wl.round_to(kb, "bf16"), wl.round_to(vb, "bf16")
    pk.kv_append(pool, torch.from_numpy(slots_b[32:]).cuda(), to_torch(kb, "bf16"),
                 to_torch(vb, "bf16"))
    q = wl.round_to(wl.prompt_queries(cfg, 0, 1, 3), "bf16")
    tables, lens, _ = pk.bt_export(pool, [1], 3)
    out = pk.paged_prefill_attention(pool, to_torch(q, "bf16"),
                                     torch.tensor([0, 3], dtype=torch.int32, device="cuda"),
                                     torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(),
                                     cfg.scale, kernel=kernel)
    torch.cuda.synchronize()
    from oracle.attention import prefill_attention
    kh = np.concatenate([to_f64(k[:32], "bf16"), to_f64(kb, "bf16")])
    vh = np.concatenate([to_f64(v[:32], "bf16"), to_f64(vb, "bf16")])
    ref = prefill_attention(to_f64(q, "bf16"), kh, vh, cfg.scale)
    compare_out(to_f64(from_torch(out, "bf16"), "bf16"), ref, "bf16")


@pytest.mark.parametrize("kernel", KERNELS)
def test_prefill_invalid_inputs(kernel):
    pool = pk.kv_pool_create(8, 16, 2, 64, "f16")
    q = torch.randn(6, 4, 64, device="cuda", dtype=torch.float16)
    tables = torch.tensor([[0, 1], [2, 3]], dtype=torch.int32, device="cuda")
    starts = torch.tensor([0, 3, 6], dtype=torch.int32, device="cuda")
    lens = torch.tensor([2, 20], dtype=torch.int32, device="cuda")        # 3 prompt rows > 2 cached
    out = pk.paged_prefill_attention(pool, q, starts, tables, lens, 0.1, kernel=kernel)
    assert pk.pkv_device_error(pool) & pk.PKV_DEVERR_CONTEXT_LEN
    assert torch.all(out[:3] == 0)
    tables = torch.tensor([[0, 1], [2, 77]], dtype=torch.int32, device="cuda")
    lens = torch.tensor([3, 20], dtype=torch.int32, device="cuda")
    out = pk.paged_prefill_attention(pool, q, starts, tables, lens, 0.1, kernel=kernel)
    assert pk.pkv_device_error(pool) & pk.PKV_DEVERR_BLOCK_ID
    assert torch.all(out[3:] == 0)
    with pytest.raises(pk.PagedKVError):                                 # f32 pool
        p32 = pk.kv_pool_create(8, 16, 2, 64, "f32")
        pk.paged_prefill_attention(p32, q.float(), starts, tables, lens, 0.1)
    with pytest.raises(pk.PagedKVError):                                 # q dtype mismatch
        pk.paged_prefill_attention(pool, q.bfloat16(), starts, tables, lens, 0.1)


@pytest.mark.parametrize("kernel", KERNELS)
def test_prefill_negative_scale(kernel):
    # the scale is a parameter (any finite value): with a negative one the
    # largest scaled score comes from the smallest raw score
    cfg = small("llama2_70b", n_q_heads=8, n_kv_heads=2, head_dim=128, kv_dtype="bf16",
                q_dtype="bf16", block_size=16, batch=3, lengths=("uniform", 150, 400))
    cfg = dataclasses.replace(cfg)
    side = setup_config(cfg, seed=21)
    hist = [side.orc.bm.lengths[s] for s in side.seqs]
    seqs = side.seqs
    qs = [wl.round_to(wl.prompt_queries(cfg, 0, s, int(n)), "bf16") for s, n in zip(seqs, hist)]
    starts = np.concatenate([[0], np.cumsum(hist)]).astype(np.int32)
    max_blocks = max(pk.bt_num_blocks(side.pool, s) for s in seqs)
    tables, lens, _ = pk.bt_export(side.pool, seqs, max_blocks)
    out = pk.paged_prefill_attention(side.pool, to_torch(np.concatenate(qs), "bf16"),
                                     torch.from_numpy(starts).cuda(),
                                     torch.from_numpy(tables).cuda(),
                                     torch.from_numpy(lens).cuda(), -cfg.scale, kernel=kernel)
    torch.cuda.synchronize()
    assert pk.pkv_device_error(side.pool) == 0
    got = to_f64(from_torch(out, "bf16"), "bf16")
    for i, (s, q) in enumerate(zip(seqs, qs)):
        ref = side.orc.prefill(s, q, "bf16", -cfg.scale)
        compare_out(got[starts[i]:starts[i + 1]], ref, "bf16")


@pytest.mark.slow
def test_prefill_full_size_sampled_rows():
    # the prompt-phase workload bench.py --mode prefill times, at full size
    # (64 sequences of the Llama-2-70B-shaped layer, every history one
    # prompt, the tcgen05 kernel): three rows per sequence - its first,
    # middle and last token - every query head, against the oracle's
    # attention of that row over its causal prefix
    from oracle.attention import decode_attention

    cfg = wl.CONFIGS["llama2_70b"]
    side = setup_config(cfg, seed=11)
    seqs = side.seqs
    n = [int(side.orc.bm.lengths[s]) for s in seqs]
    qs = [wl.round_to(wl.prompt_queries(cfg, 11, s, k), cfg.q_dtype) for s, k in zip(seqs, n)]
    starts = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    max_blocks = max(pk.bt_num_blocks(side.pool, s) for s in seqs)
    tables, lens, _ = pk.bt_export(side.pool, seqs, max_blocks)
    out = pk.paged_prefill_attention(side.pool, to_torch(np.concatenate(qs), cfg.q_dtype),
                                     torch.from_numpy(starts).cuda(),
                                     torch.from_numpy(tables).cuda(),
                                     torch.from_numpy(lens).cuda(), cfg.scale,
                                     kernel=pk.PKV_PREFILL_TCGEN05)
    torch.cuda.synchronize()
    assert pk.pkv_device_error(side.pool) == 0
    got = to_f64(from_torch(out, cfg.q_dtype), cfg.q_dtype)
    for i, s in enumerate(seqs):
        kh, vh = side.orc.history(int(s))
        kd, vd = side.orc.dequant(kh, "k"), side.orc.dequant(vh, "v")
        for t in sorted({0, n[i] // 2, n[i] - 1}):
            ref = decode_attention(to_f64(qs[i][t], cfg.q_dtype), kd[:t + 1], vd[:t + 1], cfg.scale)
            compare_out(got[starts[i] + t][None], ref[None], cfg.q_dtype)
