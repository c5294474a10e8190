"""Test harness: drive the CUDA library and the CPU oracle side by side on the
same seeded inputs (from ``workloads``) and compare them.

Nothing here computes any part of the method: the CUDA path runs through the
C ABI (``pagedattention_decode_02_b200``), the expected values come from
``oracle``.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

import pagedattention_decode_02_b200 as pk
import workloads as wl
from oracle.engine import DecodeOracle, gather_rows
from oracle.numerics import to_f64

TOL = {"f32": 1e-5, "f16": 3e-3, "bf16": 1.5e-2, "fp8": 1.5e-2}
STORE_NP = {"f32": np.float32, "f16": np.float16, "bf16": np.uint16, "fp8": np.uint8}


def to_torch(a: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    """Storage-dtype numpy array (float32 / float16 / bf16 bits) -> torch tensor."""
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(device)


def from_torch(t: torch.Tensor, dtype: str) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if dtype == "bf16":
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


@dataclasses.dataclass
class Side:
    pool: pk.Pool
    orc: DecodeOracle
    cfg: wl.Config
    seed: int
    seqs: List[int]


def make_pair(cfg: wl.Config, num_blocks: int, order, seed: int = 0, k_scale: float = 1.0,
              v_scale: float = 1.0, torch_buffers: bool = False) -> Side:
    if torch_buffers:
        nbytes = pk.kv_pool_bytes(num_blocks, cfg.block_size, cfg.n_kv_heads, cfg.head_dim,
                                  cfg.kv_dtype)
        kb = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        vb = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        pool = pk.kv_pool_create(num_blocks, cfg.block_size, cfg.n_kv_heads, cfg.head_dim,
                                 cfg.kv_dtype, k_scale, v_scale, k_buf=kb, v_buf=vb)
    else:
        pool = pk.kv_pool_create(num_blocks, cfg.block_size, cfg.n_kv_heads, cfg.head_dim,
                                 cfg.kv_dtype, k_scale, v_scale)
    pk.bt_reset(pool, order)
    orc = DecodeOracle(num_blocks, cfg.block_size, cfg.n_kv_heads, cfg.head_dim, cfg.kv_dtype,
                       k_scale, v_scale, order=order)
    return Side(pool, orc, cfg, seed, [])


def admit(side: Side, seq_ids: Sequence[int], hist_lens: Sequence[int],
          prompt_of=None) -> None:
    """Admit prompts: bt_alloc + one kv_append of all prompt rows on the GPU;
    admit on the oracle."""
    cfg = side.cfg
    slots_all, k_all, v_all = [], [], []
    for s, n in zip(seq_ids, hist_lens):
        src = prompt_of(s) if prompt_of else s
        k, v = wl.history_kv(cfg, side.seed, src, int(n))
        kr, vr = wl.round_to(k, cfg.q_dtype), wl.round_to(v, cfg.q_dtype)
        slots = pk.bt_alloc(side.pool, s, int(n))
        assert slots.tolist() == side.orc.admit(s, kr, vr, cfg.q_dtype)
        slots_all.append(slots)
        k_all.append(kr)
        v_all.append(vr)
        side.seqs.append(int(s))
    slots = np.concatenate(slots_all)
    if slots.size:
        pk.kv_append(side.pool, torch.from_numpy(slots).cuda(),
                     to_torch(np.concatenate(k_all), cfg.q_dtype),
                     to_torch(np.concatenate(v_all), cfg.q_dtype))


def fork(side: Side, parent: int, child: int) -> None:
    pk.bt_fork(side.pool, parent, child)
    side.orc.fork(parent, child)
    side.seqs.append(int(child))


def step_inputs(side: Side, seqs: Sequence[int], step: int):
    cfg = side.cfg
    qs, ks, vs = [], [], []
    for s in seqs:
        q, k, v = wl.step_qkv(cfg, side.seed, s, step)
        qs.append(q)
        ks.append(k)
        vs.append(v)
    return (wl.round_to(np.stack(qs), cfg.q_dtype), wl.round_to(np.stack(ks), cfg.q_dtype),
            wl.round_to(np.stack(vs), cfg.q_dtype))


def decode_step(side: Side, seqs: Sequence[int], step: int, partition_tokens: int = 0,
                kernel: int = pk.PKV_KERNEL_AUTO, max_blocks: Optional[int] = None,
                check_heads: Optional[Sequence[int]] = None, oracle_attend: bool = True):
    """One round on both sides.  Returns (gpu out [B][H_q][d] float64, oracle out
    (all heads or check_heads) float64, info dict)."""
    cfg = side.cfg
    q, kn, vn = step_inputs(side, seqs, step)
    slots, src, dst = pk.bt_append_batch(side.pool, seqs)
    o_slots, o_pairs = side.orc.append(seqs, kn, vn, cfg.q_dtype)
    assert slots.tolist() == o_slots
    assert list(zip(src.tolist(), dst.tolist())) == o_pairs
    if max_blocks is None:
        max_blocks = max(pk.bt_num_blocks(side.pool, s) for s in seqs)
    tables, lens, _ = pk.bt_export(side.pool, seqs, max_blocks)
    rt, rl, _ = side.orc.bm.export(seqs, max_blocks)
    assert tables.tolist() == rt and lens.tolist() == rl
    if len(src):
        pk.block_copy(side.pool, torch.from_numpy(src).cuda(), torch.from_numpy(dst).cuda())
    pk.kv_append(side.pool, torch.from_numpy(slots).cuda(), to_torch(kn, cfg.q_dtype),
                 to_torch(vn, cfg.q_dtype))
    qt = to_torch(q, cfg.q_dtype)
    out = pk.paged_decode_attention(side.pool, qt, torch.from_numpy(tables).cuda(),
                                    torch.from_numpy(lens).cuda(), cfg.scale,
                                    partition_tokens=partition_tokens, kernel=kernel)
    torch.cuda.synchronize()
    assert pk.pkv_device_error(side.pool) == 0
    gpu = to_f64(from_torch(out, cfg.q_dtype), cfg.q_dtype)
    ref = None
    if oracle_attend:
        ref = side.orc.attend(seqs, q, cfg.q_dtype, cfg.scale, heads=check_heads)
    return gpu, ref, {"tables": tables, "lens": lens, "pairs": o_pairs}


def compare_out(gpu: np.ndarray, ref: np.ndarray, dtype: str, heads=None) -> float:
    g = gpu if heads is None else gpu[:, list(heads), :]
    err = float(np.max(np.abs(g - ref)))
    assert np.all(np.isfinite(g))
    assert err <= TOL[dtype], f"max abs error {err} > {TOL[dtype]}"
    return err


def pool_image(side: Side):
    kb, vb = side.pool.device_buffers()
    dt = STORE_NP[side.cfg.kv_dtype]
    return (kb.cpu().numpy().view(dt), vb.cpu().numpy().view(dt))


def check_pool_bytes(side: Side, seqs: Optional[Sequence[int]] = None) -> None:
    """Every stored row of every sequence, read through its table from the GPU
    pool, is bit-identical to the oracle's stored row."""
    kimg, vimg = pool_image(side)
    bs = side.cfg.block_size
    for s in (side.seqs if seqs is None else seqs):
        t = side.orc.bm.tables[s]
        n = side.orc.bm.lengths[s]
        kh, vh = side.orc.history(s)
        idx = np.arange(n)
        blocks = np.asarray(t)[idx // bs]
        kg = kimg[blocks, :, idx % bs, :]
        vg = vimg[blocks, :, idx % bs, :]
        assert np.array_equal(kg.view(np.uint8), kh.view(np.uint8)), f"K rows of seq {s}"
        assert np.array_equal(vg.view(np.uint8), vh.view(np.uint8)), f"V rows of seq {s}"


def setup_config(cfg: wl.Config, seed: int = 0, variant: str = "a", growth: int = 1,
                 torch_buffers: bool = False) -> Side:
    """Pool + admitted histories for one of the named workloads."""
    lens = wl.history_lengths(cfg, seed, variant)
    k_scale = v_scale = 1.0
    if cfg.samples_per_prompt > 1:
        n_prompts = len(lens)
        per = cfg.samples_per_prompt
        nb = wl.pool_blocks(dataclasses.replace(cfg, batch=n_prompts), lens, 0) + \
            cfg.batch * (-(-(growth + cfg.block_size) // cfg.block_size) + 1)
        order = wl.free_order(nb, seed, cfg.permute)
        side = make_pair(cfg, nb, order, seed, torch_buffers=torch_buffers)
        for p_i, n in enumerate(lens):
            admit(side, [p_i * per], [int(n)], prompt_of=lambda s: s // per)
            for c in range(1, per):
                fork(side, p_i * per, p_i * per + c)
        side.seqs.sort()
        return side
    if cfg.kv_dtype == "fp8":
        k_scale, v_scale = wl.fp8_scales_for(cfg, seed, lens, steps=growth)
    nb = wl.pool_blocks(cfg, lens, growth)
    order = wl.free_order(nb, seed, cfg.permute)
    side = make_pair(cfg, nb, order, seed, k_scale, v_scale, torch_buffers=torch_buffers)
    admit(side, list(range(len(lens))), [int(n) for n in lens])
    return side
