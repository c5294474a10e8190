"""Guard blocks around a pool's own K/V buffers: untouched by the library's
kernels and copies, and the check notices a changed byte (a write planted
in the guard region itself, inside the pool's allocation)."""

import numpy as np
import pytest
import torch

import pagedattention_decode_02_b200 as pk
import workloads as wl
from paged_harness import compare_out, decode_step, setup_config

pytestmark = pytest.mark.gpu


def _guard_view(ptr: int, offset: int, n: int):
    return torch.as_tensor(pk._CudaArray(ptr + offset, (n,)), device="cuda")


def test_guards_untouched_by_append_decode_and_swap():
    cfg = wl.CONFIGS["toy"]
    side = setup_config(cfg)
    for t in range(3):
        gpu, ref, _ = decode_step(side, list(range(cfg.batch)), t)
        compare_out(gpu, ref, "f32")
    blk = pk.block_bytes(side.pool)
    n = pk.bt_num_blocks(side.pool, 0)
    hk = torch.empty(n * blk, dtype=torch.uint8).pin_memory()
    hv = torch.empty(n * blk, dtype=torch.uint8).pin_memory()
    pk.kv_swap_out(side.pool, 0, hk, hv)
    torch.cuda.synchronize()
    assert pk.kv_pool_check_guards(side.pool)


def test_a_changed_guard_byte_is_reported():
    pool = pk.kv_pool_create(8, 4, 2, 64, "f16")
    assert pk.kv_pool_check_guards(pool)
    info = pool.info
    span = pool.num_blocks * pool.n_kv_heads * pool.block_size * pool.head_dim * 2
    for ptr, off in ((info.k_buf, -16), (info.v_buf, span)):
        g = _guard_view(ptr, off, 16)
        keep = g.clone()
        g.fill_(0)
        torch.cuda.synchronize()
        assert not pk.kv_pool_check_guards(pool)
        g.copy_(keep)
        torch.cuda.synchronize()
        assert pk.kv_pool_check_guards(pool)
    pool.close()


def test_caller_owned_buffers_have_no_guards():
    need = pk.kv_pool_bytes(8, 4, 2, 64, "f16")
    kb = torch.zeros(need, dtype=torch.uint8, device="cuda")
    vb = torch.zeros(need, dtype=torch.uint8, device="cuda")
    pool = pk.kv_pool_create(8, 4, 2, 64, "f16", k_buf=kb, v_buf=vb)
    assert pk.kv_pool_check_guards(pool)
    pool.close()
