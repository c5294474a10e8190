"""The decode-step runtime's prefetch block.  For each launch slot the host
passes the context length, the table row and how many leading entries of
that row the round's prologue leaves as they are; the decode kernel loads
those entries, and the stages whose blocks they cover, before the prologue
has finished, and the rest after it.  Checked against the oracle round by
round:

* with the boundary between kept and updated entries falling inside
  partitions (partitions of 16 and 48 tokens, and unsplit) at block sizes
  1, 4 and 16, on the CUDA-core kernel, the tensor-core kernel and its FP8
  form;
* after copy-on-write of a shared last block (samples of one prompt);
* with more launch slots than the block covers (the kernel then takes
  every length, row and entry from the prologue's output).
"""

import dataclasses

import numpy as np
import pytest

import pagedattention_decode_02_b200 as pk
import workloads as wl
from paged_harness import check_pool_bytes, setup_config
from test_gpu_step import run_rounds

pytestmark = pytest.mark.gpu

# kernel, query / KV heads, pool dtype
CASES = {
    "simt2": (pk.PKV_KERNEL_SIMT_TMA, 4, 4, "f16"),
    "tensor": (pk.PKV_KERNEL_TENSOR, 16, 2, "f16"),
    "tensor_fp8": (pk.PKV_KERNEL_TENSOR, 4, 4, "fp8"),
}


@pytest.mark.parametrize("partition", [16, 48, 0])
@pytest.mark.parametrize("bs", [1, 4, 16])
@pytest.mark.parametrize("case", sorted(CASES))
def test_kept_entries_boundary_with_copy_on_write(case, bs, partition):
    kernel, hq, hkv, kv = CASES[case]
    # 2 prompts x 4 samples: every sample's first append copies the shared
    # last block, and the kept entries end just before it
    cfg = dataclasses.replace(wl.CONFIGS["falcon7b"], n_q_heads=hq, n_kv_heads=hkv, head_dim=128,
                              kv_dtype=kv, block_size=bs, batch=8, lengths=("fixed", 300))
    side = setup_config(cfg, variant="b", growth=20)
    run_rounds(cfg, side, 20, partition=partition, kernel=kernel)
    check_pool_bytes(side)
    # (prompts of 293 tokens: with one token per block nothing is shared)
    assert (pk.bt_stats(side.pool)["cow_count"] > 0) == (bs > 1)


def test_more_launch_slots_than_the_block_covers():
    # 140 sequences: the parameter-block path still holds the round, the
    # prefetch block (128 slots) is left empty
    cfg = dataclasses.replace(wl.CONFIGS["opt13b"], n_q_heads=2, n_kv_heads=2, batch=140,
                              lengths=("uniform", 1, 90), min_pool_blocks=0)
    side = setup_config(cfg, growth=6)
    run_rounds(cfg, side, 6, kernel=pk.PKV_KERNEL_SIMT_TMA)
    check_pool_bytes(side)

