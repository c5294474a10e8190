"""The tcgen05 prompt kernel's run-time work schedule: CTAs claim work items
from a pair of counters kept in the pool (one pair per launch in flight,
taken in turn from 64; the launch's last CTA zeroes its pair).  Checked
against the oracle:

* more launches on one pool than there are counter pairs, each result
  bit-identical to the first (every pair reused comes back zeroed);
* two launches queued on two streams at once (different pairs, no
  ordering between them);
* a batch of more sequences than the kernel keeps the group-major order
  for in shared memory (the rank-major order, in which most claimed item
  indices hold no work).
"""

import dataclasses

import numpy as np
import pytest
import torch

import pagedattention_decode_02_b200 as pk
import workloads as wl
from paged_harness import compare_out, from_torch, setup_config, to_torch
from oracle.numerics import to_f64

pytestmark = pytest.mark.gpu

K = pk.PKV_PREFILL_TCGEN05


def _batch(cfg, seed):
    side = setup_config(cfg, seed=seed)
    seqs = side.seqs
    n = [int(side.orc.bm.lengths[s]) for s in seqs]
    qs = [wl.round_to(wl.prompt_queries(cfg, seed, s, k), cfg.q_dtype) for s, k in zip(seqs, n)]
    starts = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    max_blocks = max(pk.bt_num_blocks(side.pool, s) for s in seqs)
    tables, lens, _ = pk.bt_export(side.pool, seqs, max_blocks)
    dev = (to_torch(np.concatenate(qs), cfg.q_dtype), torch.from_numpy(starts).cuda(),
           torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda())
    return side, qs, starts, dev


def _check(side, qs, starts, out, cfg, every=1):
    got = to_f64(from_torch(out, cfg.q_dtype), cfg.q_dtype)
    for i in range(0, len(qs), every):
        ref = side.orc.prefill(side.seqs[i], qs[i], cfg.q_dtype, cfg.scale)
        compare_out(got[starts[i]:starts[i + 1]], ref, cfg.q_dtype)


def test_more_launches_than_counter_pairs():
    cfg = dataclasses.replace(wl.CONFIGS["llama2_70b"], n_q_heads=16, n_kv_heads=2, batch=6,
                              lengths=("uniform", 100, 600))
    side, qs, starts, (q, st, tb, ln) = _batch(cfg, seed=3)
    first = pk.paged_prefill_attention(side.pool, q, st, tb, ln, cfg.scale, kernel=K)
    torch.cuda.synchronize()
    assert pk.pkv_device_error(side.pool) == 0
    _check(side, qs, starts, first, cfg)
    out = torch.empty_like(q)
    for i in range(150):                      # > 2 x 64 pairs
        pk.paged_prefill_attention(side.pool, q, st, tb, ln, cfg.scale, out=out, kernel=K)
        if i % 37 == 0 or i == 149:
            torch.cuda.synchronize()
            assert torch.equal(out, first), i
    assert pk.pkv_device_error(side.pool) == 0


def test_two_streams_at_once():
    cfg = dataclasses.replace(wl.CONFIGS["llama2_70b"], n_q_heads=8, n_kv_heads=2, batch=5,
                              lengths=("uniform", 200, 900))
    side, qs, starts, (q, st, tb, ln) = _batch(cfg, seed=4)
    # a second query batch over the same pool
    n = np.diff(starts)
    qs2 = [wl.round_to(wl.prompt_queries(cfg, 40, s, int(k)), cfg.q_dtype)
           for s, k in zip(side.seqs, n)]
    q2 = to_torch(np.concatenate(qs2), cfg.q_dtype)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(s1):
        o1 = pk.paged_prefill_attention(side.pool, q, st, tb, ln, cfg.scale, stream=s1, kernel=K)
    with torch.cuda.stream(s2):
        o2 = pk.paged_prefill_attention(side.pool, q2, st, tb, ln, cfg.scale, stream=s2, kernel=K)
    torch.cuda.synchronize()
    assert pk.pkv_device_error(side.pool) == 0
    _check(side, qs, starts, o1, cfg)
    _check(side, qs2, starts, o2, cfg)


def test_many_sequences_rank_major_order():
    # more sequences than the group-major order is kept for (1024): items
    # are numbered rank-major and most claimed indices hold no work
    cfg = dataclasses.replace(wl.CONFIGS["llama2_70b"], n_q_heads=4, n_kv_heads=2, head_dim=64,
                              batch=1100, lengths=("uniform", 1, 300))
    side, qs, starts, (q, st, tb, ln) = _batch(cfg, seed=5)
    out = pk.paged_prefill_attention(side.pool, q, st, tb, ln, cfg.scale, kernel=K)
    torch.cuda.synchronize()
    assert pk.pkv_device_error(side.pool) == 0
    _check(side, qs, starts, out, cfg, every=7)
