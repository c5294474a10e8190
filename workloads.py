"""Seeded synthetic inputs for the paged decode step.

This module is shared by the CUDA path's tests, ``bench.py``, ``smoke()`` and
the CPU oracle's tests.  It holds random draws, the rounding of those draws to
the storage dtype the caller asked for, and the sizing of the synthetic batches.
It holds none of the method's arithmetic: no attention, no block-table logic,
no FP8 quantisation.

Workload shapes follow the pages' workloads (KV 缓存与分页注意力, §一个词元
800 KB, §快了多少, §后来的做法, §实验台; the ShareGPT/Alpaca request mixes they
quote are not available, so lengths are drawn from the distributions below):

* ``toy``        - the exhibit's machine: 44 physical blocks of 4 slots, one head,
                   head_dim 32, fp32; 6 sequences, history length U{1..20}.
* ``opt13b``     - one OPT-13B layer: 40 MHA heads x 128, fp16, block 16; 30
                   sequences (the quoted mean batch), history U{64..2048}; pool
                   of max(982, needed) blocks (982 x 16 = the quoted ~15,700 tokens).
* ``llama2_70b`` - one Llama-2-70B layer: 64 q heads on 8 KV heads x 128, bf16,
                   block 16; 64 sequences, history floor(exp U[ln 128, ln 4096]).
* ``falcon7b``   - Falcon-7B MQA: 71 q heads on 1 KV head x 64, fp16, block 16;
                   16 prompts x 4 samples; prompts of 512 tokens (variant "a") or
                   512 - r, r ~ U{1..15} (variant "b"); 64 decode steps.
* ``fp8``        - the OPT-13B layer with an FP8-E4M3 pool, fp16 q/out; 128
                   sequences, history U{1..2048}; block size swept 1..64.

All draws come from ``numpy.random.default_rng`` seeded with a tuple
``(seed, stream tag, ids...)`` so that any single sequence's data can be
regenerated on its own.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

# stream tags for default_rng seed tuples
_TAG_LENGTHS = 1
_TAG_ORDER = 2
_TAG_HIST_K = 3
_TAG_HIST_V = 4
_TAG_STEP = 5
_TAG_PROMPT_R = 6

DTYPES = ("f32", "f16", "bf16", "fp8")
ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2, "fp8": 1}


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    kv_dtype: str          # storage dtype of the pool
    q_dtype: str           # dtype of q, of the new K/V rows and of the output
    block_size: int
    batch: int
    lengths: tuple         # ("uniform", lo, hi) | ("loguniform", lo, hi) | ("fixed", n)
    min_pool_blocks: int = 0
    permute: bool = True
    samples_per_prompt: int = 1
    steps: int = 1
    description: str = ""

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def kv_bytes_per_token(self) -> int:
        """b_tok = 2 * H_kv * d * bytes: one layer's K and V for one token."""
        return 2 * self.n_kv_heads * self.head_dim * ELEM_BYTES[self.kv_dtype]

    def with_block_size(self, bs: int) -> "Config":
        return dataclasses.replace(self, block_size=bs)


CONFIGS = {
    "toy": Config(
        "toy", 1, 1, 32, "f32", "f32", 4, 6, ("uniform", 1, 20),
        min_pool_blocks=44, permute=False,
        description="exhibit machine: 44 blocks x 4 slots, 1 head, d 32, fp32, 6 seqs"),
    "opt13b": Config(
        "opt13b", 40, 40, 128, "f16", "f16", 16, 30, ("uniform", 64, 2048),
        min_pool_blocks=982, permute=True,
        description="OPT-13B layer: 40x128 MHA fp16, bs 16, 30 seqs, history U[64,2048]"),
    "llama2_70b": Config(
        "llama2_70b", 64, 8, 128, "bf16", "bf16", 16, 64, ("loguniform", 128, 4096),
        permute=True,
        description="Llama-2-70B layer: 64/8 GQA x128 bf16, bs 16, 64 seqs, history log-U[128,4096]"),
    "falcon7b": Config(
        "falcon7b", 71, 1, 64, "f16", "f16", 16, 64, ("fixed", 512),
        permute=True, samples_per_prompt=4, steps=64,
        description="Falcon-7B MQA: 71/1 x64 fp16, bs 16, 16 prompts x 4 samples, 64 steps"),
    "fp8": Config(
        "fp8", 40, 40, 128, "fp8", "f16", 16, 128, ("uniform", 1, 2048),
        permute=True,
        description="OPT-13B layer, FP8-E4M3 pool, fp16 q/out, 128 seqs, history U[1,2048]"),
    "fp8_gqa": Config(
        "fp8_gqa", 64, 8, 128, "fp8", "f16", 16, 64, ("loguniform", 128, 4096),
        permute=True,
        description="Llama-2-70B layer, FP8-E4M3 pool, fp16 q/out: 64/8 GQA x128, bs 16, "
                    "64 seqs, history log-U[128,4096]"),
}

FP8_BLOCK_SIZES = (1, 2, 4, 8, 16, 32, 64)


def _rng(seed: int, *ids: int) -> np.random.Generator:
    return np.random.default_rng([int(seed)] + [int(i) for i in ids])


# ---------------------------------------------------------------------------
# lengths, pool sizes, block orders
# ---------------------------------------------------------------------------

def history_lengths(cfg: Config, seed: int = 0, variant: str = "a") -> np.ndarray:
    """Cached tokens per sequence *before* the decode step's append.

    For ``falcon7b`` this is one entry per prompt (16), not per sample.
    """
    kind = cfg.lengths[0]
    if cfg.samples_per_prompt > 1:
        n_prompts = cfg.batch // cfg.samples_per_prompt
        base = np.full(n_prompts, cfg.lengths[1], dtype=np.int64)
        if variant == "b":
            r = _rng(seed, _TAG_PROMPT_R).integers(1, 16, size=n_prompts)
            base = base - r
        return base
    g = _rng(seed, _TAG_LENGTHS)
    if kind == "uniform":
        return g.integers(cfg.lengths[1], cfg.lengths[2] + 1, size=cfg.batch).astype(np.int64)
    if kind == "loguniform":
        u = g.uniform(math.log(cfg.lengths[1]), math.log(cfg.lengths[2]), size=cfg.batch)
        return np.floor(np.exp(u)).astype(np.int64)
    if kind == "fixed":
        return np.full(cfg.batch, cfg.lengths[1], dtype=np.int64)
    raise ValueError(kind)


def pool_blocks(cfg: Config, hist_lengths, growth: int = 1) -> int:
    """Physical blocks for a batch: room for every history plus ``growth`` more
    tokens per sequence, plus one spare block per sequence (copy-on-write or a
    fresh block on the next append), and at least ``cfg.min_pool_blocks``."""
    bs = cfg.block_size
    need = int(sum((int(n) + growth + bs - 1) // bs for n in hist_lengths))
    need += cfg.batch
    return max(cfg.min_pool_blocks, need)


def free_order(num_blocks: int, seed: int = 0, permute: bool = True) -> np.ndarray:
    """Initial order of the free-block queue: identity (blocks handed out in
    arrival order) or a seeded random permutation of the physical ids."""
    if not permute:
        return np.arange(num_blocks, dtype=np.int32)
    return _rng(seed, _TAG_ORDER).permutation(num_blocks).astype(np.int32)


# ---------------------------------------------------------------------------
# values
# ---------------------------------------------------------------------------

def history_kv(cfg: Config, seed: int, seq: int, n: int):
    """K and V rows of one sequence's history (or one prompt's, for ``falcon7b``):
    float32 N(0,1), shape [n][H_kv][d]."""
    shape = (int(n), cfg.n_kv_heads, cfg.head_dim)
    k = _rng(seed, _TAG_HIST_K, seq).standard_normal(shape, dtype=np.float32)
    v = _rng(seed, _TAG_HIST_V, seq).standard_normal(shape, dtype=np.float32)
    return k, v


def step_qkv(cfg: Config, seed: int, seq: int, step: int):
    """q [H_q][d], new k and v [H_kv][d] of one sequence at one decode step,
    float32 N(0,1)."""
    g = _rng(seed, _TAG_STEP, seq, step)
    q = g.standard_normal((cfg.n_q_heads, cfg.head_dim), dtype=np.float32)
    k = g.standard_normal((cfg.n_kv_heads, cfg.head_dim), dtype=np.float32)
    v = g.standard_normal((cfg.n_kv_heads, cfg.head_dim), dtype=np.float32)
    return q, k, v


def prompt_queries(cfg: Config, seed: int, seq: int, n: int) -> np.ndarray:
    """Queries of a sequence's last n prompt tokens: [n][H_q][d] float32, N(0,1)."""
    rng = _rng(seed, 7, seq, n)
    return rng.standard_normal((n, cfg.n_q_heads, cfg.head_dim), dtype=np.float32)


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 draws to a storage dtype (round to nearest even).

    Returns float32 for "f32", float16 for "f16" and the raw uint16 bit patterns
    for "bf16" (numpy has no bfloat16).
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f32":
        return x
    if dtype == "f16":
        return x.astype(np.float16)
    if dtype == "bf16":
        b = x.view(np.uint32).astype(np.uint64)
        b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
        return b.astype(np.uint16)
    raise ValueError(dtype)


def fp8_scale(amax: float) -> float:
    """Per-tensor FP8-E4M3 scale that maps amax onto the largest finite code
    (448), rounded to float32."""
    return float(np.float32(np.float32(amax) / np.float32(448.0)))


def fp8_scales_for(cfg: Config, seed: int, hist_lengths, steps: int = 1):
    """(k_scale, v_scale) from the amax of every K (resp. V) row the run will
    write: histories and the ``steps`` decode steps' new rows, all rounded to
    ``cfg.q_dtype`` first (the dtype the rows are handed over in)."""
    ka = 0.0
    va = 0.0
    for i, n in enumerate(hist_lengths):
        k, v = history_kv(cfg, seed, i, int(n))
        ka = max(ka, float(np.abs(_as_f32(round_to(k, cfg.q_dtype), cfg.q_dtype)).max(initial=0.0)))
        va = max(va, float(np.abs(_as_f32(round_to(v, cfg.q_dtype), cfg.q_dtype)).max(initial=0.0)))
        for t in range(steps):
            _, kn, vn = step_qkv(cfg, seed, i, t)
            ka = max(ka, float(np.abs(_as_f32(round_to(kn, cfg.q_dtype), cfg.q_dtype)).max()))
            va = max(va, float(np.abs(_as_f32(round_to(vn, cfg.q_dtype), cfg.q_dtype)).max()))
    return fp8_scale(ka), fp8_scale(va)


def _as_f32(a: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return (a.astype(np.uint32) << 16).view(np.float32)
    return a.astype(np.float32)


def seq_ids(cfg: Config) -> np.ndarray:
    return np.arange(cfg.batch, dtype=np.int64)


def prompt_of(cfg: Config, seq: int) -> int:
    return int(seq) // cfg.samples_per_prompt


def bytes_per_step(cfg: Config, context_lens) -> int:
    """Algorithmic KV bytes one decode step reads: sum_i c_i * b_tok."""
    return int(np.sum(np.asarray(context_lens, dtype=np.int64))) * cfg.kv_bytes_per_token


def describe(cfg: Config, seed: int = 0, variant: Optional[str] = None) -> dict:
    d = dataclasses.asdict(cfg)
    d["seed"] = seed
    if variant:
        d["variant"] = variant
    return d


# ---------------------------------------------------------------------------
# the exhibit's allocation bench
# ---------------------------------------------------------------------------

EXHIBIT_SLOTS = 176      # 44 blocks of 4 token slots
EXHIBIT_MAX_LEN = 20     # longest sequence, tokens
EXHIBIT_MODES = (1, 2, 4, 8, 16, 0)   # block sizes, and 0 for the max-length reservation


def exhibit_requests(n: int, seed: int = 0, per_round: int = 2, max_len: int = EXHIBIT_MAX_LEN):
    """n requests (arrival round, prompt, output), per_round arriving each
    round; final length uniform on [2, max_len], prompt uniform on [1, length-1]
    (the exhibit draws lengths at random, not from a trace)."""
    rng = _rng(seed, 4242, n, per_round)
    total = rng.integers(2, max_len + 1, size=n)
    prompt = np.array([rng.integers(1, t) for t in total], dtype=np.int64)
    return [(i // per_round, int(p), int(t - p)) for i, (p, t) in enumerate(zip(prompt, total))]
