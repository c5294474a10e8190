"""GPU parity of the exact path bench.py times, at full size.

bench.py times the decode-step runtime (pkv_decode_step: host block-table
update, the prologue kernel with copy-on-write and append, the automatic
decode kernel with its in-kernel split merge, programmatic dependent launch,
persistent device table rows with least-recently-used eviction, longest-first
launch order) on several replica batches of a workload held in one pool, with
max_seqs = batch x replicas.  This test builds the same pool the same way -
replica batch r has the workload's lengths for seed r, ids r*B .. r*B+B-1, the
pool sized by the bench's formula (room for the rounds run), the free queue a seeded permutation - but
with histories drawn by the seeded numpy generator, so that the oracle holds
the same values.  It then runs two rounds per replica batch in the bench's
order (the first round of a batch uploads its tables, the second travels as
kernel parameters) and compares EVERY query head of EVERY sequence with the
oracle after each round ("KV 缓存与分页注意力" §一次写一个词元, §块表), within
the stated tolerance (fp16 3e-3, bf16 1.5e-2).
"""

import numpy as np
import pytest
import torch

import pagedattention_decode_02_b200 as pk
import workloads as wl
from bench import auto_replicas
from oracle.numerics import to_f64
from paged_harness import TOL, admit, compare_out, from_torch, make_pair, step_inputs, to_torch

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

ROUNDS_PER_BATCH = 2


def build_replicas(cfg: wl.Config, R: int, growth: int):
    """The bench's pool of R replica batches, with oracle-visible histories."""
    B = cfg.batch
    lens = [wl.history_lengths(cfg, r, "b") for r in range(R)]
    nb = sum(wl.pool_blocks(cfg, l, growth) for l in lens)
    side = make_pair(cfg, nb, wl.free_order(nb, 0, cfg.permute), seed=0)
    groups = []
    for r in range(R):
        side.seed = r                      # replica r's histories: seed r, as its lengths
        ids = [r * B + i for i in range(B)]
        admit(side, ids, [int(n) for n in lens[r]], prompt_of=lambda s: s % B)
        groups.append(np.asarray(ids, dtype=np.int64))
    side.seed = 0                          # decode-round inputs: seeded per global id
    max_ctx = max(int(l.max()) for l in lens) + growth
    return side, groups, -(-max_ctx // cfg.block_size) + 2


@pytest.mark.parametrize("name", ["opt13b", "llama2_70b"])
def test_timed_path_full_size_every_head(name):
    cfg = wl.CONFIGS[name]
    R = auto_replicas(cfg)
    assert R >= 8
    growth = ROUNDS_PER_BATCH + 2
    side, groups, max_blocks = build_replicas(cfg, R, growth)
    B = cfg.batch
    step = pk.Step(side.pool, B, max_blocks, cfg.n_q_heads, cfg.q_dtype, 0, 0, max_seqs=B * R)
    out = torch.empty((B, cfg.n_q_heads, cfg.head_dim), device="cuda",
                      dtype={"f16": torch.float16, "bf16": torch.bfloat16}[cfg.q_dtype])
    tol_dtype = cfg.q_dtype
    kernels = set()
    worst = 0.0
    for k in range(ROUNDS_PER_BATCH * R):
        r = k % R
        seqs = groups[r]
        q, kn, vn = step_inputs(side, seqs, k // R)
        pk.pkv_decode_step(step, seqs, to_torch(q, cfg.q_dtype), to_torch(kn, cfg.q_dtype),
                           to_torch(vn, cfg.q_dtype), cfg.scale, out)
        kernels.add(step.last_kernel)
        side.orc.append(list(seqs), kn, vn, cfg.q_dtype)
        ref = side.orc.attend(list(seqs), q, cfg.q_dtype, cfg.scale)     # every head
        torch.cuda.synchronize()
        gpu = to_f64(from_torch(out, cfg.q_dtype), cfg.q_dtype)
        worst = max(worst, compare_out(gpu, ref, tol_dtype))
    assert pk.pkv_device_error(side.pool) == 0
    assert len(kernels) == 1 and 0 not in kernels
    print(f"{name}: {2 * R} rounds x {B} seqs x {cfg.n_q_heads} heads, kernel "
          f"{pk.KERNEL_NAMES[kernels.pop()]}, max abs error {worst:.3e} (tol {TOL[tol_dtype]})")
