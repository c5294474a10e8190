"""The decode entry point that allocates nothing (paged_decode_attention_static).

Some callers cannot call cudaMalloc: a process whose device memory is already
held by another allocator, or a latency-bound loop that allows no
cudaMalloc/cudaFree after warm-up because they can synchronise the device.
For them the split-context scratch is a static device array inside the
library.  These tests call that entry point through the C ABI and check it
against the regular entry point (which takes a caller-allocated workspace) on
the same inputs, on consecutive calls.  The file sorts last so that a run
stopping at the first failure has already run every other test; it also
passes on its own in a fresh process (the first call does the per-device
set-up).
"""

import dataclasses

import numpy as np
import pytest
import torch

import pagedattention_decode_02_b200 as pk
import workloads as wl
from oracle.numerics import to_f64
from paged_harness import TOL, from_torch, setup_config, step_inputs, to_torch

pytestmark = pytest.mark.gpu


def _prepared_batch(cfg, seed):
    side = setup_config(cfg, seed=seed)
    seqs = list(range(cfg.batch))
    q, kn, vn = step_inputs(side, seqs, 0)
    slots, src, dst = pk.bt_append_batch(side.pool, seqs)
    side.orc.append(seqs, kn, vn, cfg.q_dtype)
    pk.kv_append(side.pool, torch.from_numpy(slots).cuda(), to_torch(kn, cfg.q_dtype),
                 to_torch(vn, cfg.q_dtype))
    max_blocks = max(pk.bt_num_blocks(side.pool, s) for s in seqs)
    tables, lens, _ = pk.bt_export(side.pool, seqs, max_blocks)
    return side, seqs, to_torch(q, cfg.q_dtype), q, torch.from_numpy(tables).cuda(), \
        torch.from_numpy(lens).cuda()


@pytest.mark.parametrize("base,dt", [("opt13b", "f16"), ("llama2_70b", "bf16")])
def test_static_scratch_matches_the_workspace_entry_point(base, dt):
    cfg = dataclasses.replace(wl.CONFIGS[base], n_q_heads=8, n_kv_heads=8 if base == "opt13b" else 2,
                              batch=12, lengths=("uniform", 600, 2000), min_pool_blocks=0)
    side, seqs, qt, q, tables, lens = _prepared_batch(cfg, seed=5)
    # the batch is long enough to be split, so the scratch is really used
    assert pk.paged_decode_workspace_bytes(side.pool, cfg.batch, cfg.n_q_heads,
                                           tables.shape[1]) > 0
    ref = pk.paged_decode_attention(side.pool, qt, tables, lens, cfg.scale)
    torch.cuda.synchronize()
    expect = side.orc.attend(seqs, q, cfg.q_dtype, cfg.scale)
    for _ in range(2):        # two calls in a row share the static scratch
        out = torch.full_like(qt, float("nan"))
        pk.paged_decode_attention_static(side.pool, qt, tables, lens, cfg.scale, out=out)
        torch.cuda.synchronize()
        got = to_f64(from_torch(out, cfg.q_dtype), cfg.q_dtype)
        base_out = to_f64(from_torch(ref, cfg.q_dtype), cfg.q_dtype)
        assert np.all(np.isfinite(got))
        assert np.max(np.abs(got - base_out)) <= TOL[cfg.q_dtype]
        assert np.max(np.abs(got - expect)) <= TOL[cfg.q_dtype]
    assert pk.pkv_device_error(side.pool) == 0


def test_static_scratch_limit_is_reported_without_launching():
    cfg = dataclasses.replace(wl.CONFIGS["opt13b"], batch=30, lengths=("uniform", 1900, 2000))
    side, seqs, qt, q, tables, lens = _prepared_batch(cfg, seed=6)
    need = pk.paged_decode_workspace_bytes(side.pool, 30, 40, tables.shape[1], partition_tokens=16)
    assert need > pk.paged_decode_static_scratch_bytes()
    out = torch.zeros_like(qt)
    with pytest.raises(pk.PagedKVError) as e:
        pk.paged_decode_attention_static(side.pool, qt, tables, lens, cfg.scale, out=out,
                                         partition_tokens=16)
    assert e.value.status == pk.PKV_ERR_SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert torch.all(out == 0)
    # automatic partitioning never exceeds the scratch: it picks longer partitions
    pk.paged_decode_attention_static(side.pool, qt, tables, lens, cfg.scale, out=out)
    torch.cuda.synchronize()
    got = to_f64(from_torch(out, "f16"), "f16")
    heads = [0, 17, 39]
    expect = side.orc.attend(seqs, q, "f16", cfg.scale, heads=heads)
    assert np.max(np.abs(got[:, heads, :] - expect)) <= TOL["f16"]
