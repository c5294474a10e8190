"""Host-side partition choice and bench bookkeeping (no GPU needed).

The automatic partitioning is observable through the workspace the library
asks for: a batch whose unsplit grid already has two waves of CTAs (three per
SM, 148 SMs when the device is unknown) is not split and needs none; smaller
batches with long contexts are split into partitions of 512 tokens (one head
per KV head) or 1536 tokens per 8 grouped heads, each partition leaving
(d + 2) floats per query head in the workspace."""

import pytest

import pagedattention_decode_02_b200 as pk
import workloads as wl

def _rows_floats(B, Hq, parts, d):
    rows = B * Hq * parts
    ml = (rows * 2 * 4 + 255) & ~255
    return ml + rows * d * 4


def test_unsplit_when_the_batch_fills_two_waves():
    p = pk.kv_pool_create(64, 16, 40, 128, "f16", host_only=True)
    max_blocks = 130                                   # contexts up to 2,080 tokens
    # 30 sequences x 40 heads = 1,200 CTAs >= 2 x 3 x 148: no split, no workspace
    assert pk.paged_decode_workspace_bytes(p, 30, 40, max_blocks) == 0
    # 2 sequences x 40 heads: split into ceil(2080 / 512) = 5 partitions
    assert pk.paged_decode_workspace_bytes(p, 2, 40, max_blocks) == _rows_floats(2, 40, 5, 128)
    # an explicit partition is taken as given
    assert pk.paged_decode_workspace_bytes(p, 30, 40, max_blocks, 512) == \
        _rows_floats(30, 40, 5, 128)
    # -1 never splits
    assert pk.paged_decode_workspace_bytes(p, 2, 40, max_blocks, -1) == 0


def test_grouped_heads_take_1536_token_partitions():
    p = pk.kv_pool_create(64, 16, 8, 128, "bf16", host_only=True)
    max_blocks = 260                                   # 4,160 tokens -> 3 partitions of 1536
    # 64 sequences x 8 KV heads = 512 CTAs < 888: split
    assert pk.paged_decode_workspace_bytes(p, 64, 64, max_blocks) == _rows_floats(64, 64, 3, 128)
    # 16 query heads per KV head: 3072-token partitions -> 2 (32 x 8 x 2 = 512 CTAs)
    assert pk.paged_decode_workspace_bytes(p, 32, 128, max_blocks) == _rows_floats(32, 128, 2, 128)
    # ... and 64 sequences already fill two waves (64 x 8 x 2 = 1,024 CTAs)
    assert pk.paged_decode_workspace_bytes(p, 64, 128, max_blocks) == 0
    # contexts up to 512 tokens are never split
    assert pk.paged_decode_workspace_bytes(p, 4, 64, 32) == 0


def test_bench_cycles_more_kv_than_three_l2s():
    import bench
    for name in ("opt13b", "llama2_70b", "falcon7b", "fp8", "fp8_gqa"):
        cfg = wl.CONFIGS[name]
        r = bench.auto_replicas(cfg)
        assert r >= 8
        assert r * bench.distinct_kv_bytes(cfg) >= 3 * bench.L2_BYTES


def test_bench_traffic_only_at_the_captured_block_size():
    import bench
    cfg = wl.CONFIGS["fp8"]
    assert bench.traffic_per_launch(cfg.with_block_size(1), "decode_simt2_kernel", 1e9) is None
    assert bench.traffic_per_launch(cfg, "no_such_kernel", 1e9) is None


def test_bench_roofline_recomputes_from_its_own_fields():
    # achieved = profiled_bytes / (profiled_launches x decode_ms_mean), and
    # frac = achieved / peak, from the printed fields alone
    import bench
    cfg = wl.CONFIGS["opt13b"]
    m = {"kernel": "decode_simt2_kernel", "dec_ms": [0.110, 0.108, 0.112],
         "prof_bytes": [605_000_000, 604_000_000, 606_000_000],
         "step_bytes": [605_000_000] * 9, "merge_ms": [0.0, 0.0, 0.0],
         "pro_ms": [0.007, 0.008, 0.0075], "prof_batches": [0, 1, 2], "prof_every": 3, "R": 8}
    r = bench.roofline_of(cfg, m, 6650.0, "fallback")
    n = r["profiled_launches"]
    assert n == 3 and r["profiled_bytes"] == sum(m["prof_bytes"])
    achieved = r["profiled_bytes"] / n / (r["decode_ms_mean"] / 1e3) / 1e9
    assert abs(achieved - r["achieved"]) <= 0.01 * achieved
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-4
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
