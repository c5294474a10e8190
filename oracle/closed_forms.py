"""Closed forms the pages fix.  TEST INFRASTRUCTURE ONLY.

* Per-token KV bytes ("KV 缓存与分页注意力", §一个词元 800 KB; the "KV 缓存" topic
  page, level 1 formula): every token has one key and one value per layer, so
  bytes = 2 x layers x H_kv x d_head x bytes_per_element; the batch-wide form
  multiplies by B and by the number of positions N.
* Pool capacity (§一个词元 800 KB, §先占好最长的位置): KV space / per-token bytes,
  and whole max-length sequences that fit.  The exhibit's KB and GB are binary
  (§模型省略了什么).
* Utilisation (§块表, §实验台): of the slots a sequence's blocks reserve, how
  many hold tokens; with allocation only on a full block, the waste per
  sequence is below one block.
"""

from __future__ import annotations

from fractions import Fraction
from typing import Iterable, Sequence


def kv_bytes_per_token(layers: int, n_kv_heads: int, head_dim: int, bytes_per_elem: int) -> int:
    return 2 * layers * n_kv_heads * head_dim * bytes_per_elem


def kv_cache_bytes(batch: int, layers: int, positions: int, n_kv_heads: int, head_dim: int,
                   bytes_per_elem: int) -> int:
    """B x L x N x 2 x H_kv x d_head x bytes (topic page, level 1)."""
    return batch * layers * positions * 2 * n_kv_heads * head_dim * bytes_per_elem


def tokens_that_fit(kv_space_bytes: int, per_token_bytes: int) -> int:
    return kv_space_bytes // per_token_bytes


def max_length_sequences_that_fit(kv_space_bytes: int, per_token_bytes: int, max_len: int) -> int:
    return kv_space_bytes // (per_token_bytes * max_len)


def blocks_for(n_tokens: int, block_size: int) -> int:
    """Blocks a sequence of n tokens holds when a block is taken only once the
    previous one is full."""
    return -(-n_tokens // block_size)


def utilisation(context_lens: Iterable[int], block_size: int) -> Fraction:
    """sum c_i / sum(|table_i| * bs): the fraction of reserved slots that hold
    tokens (no sharing)."""
    cs = [int(c) for c in context_lens]
    reserved = sum(blocks_for(c, block_size) * block_size for c in cs)
    return Fraction(sum(cs), reserved)


def max_reservation_utilisation(context_lens: Sequence[int], max_len: int) -> Fraction:
    """The same ratio when every sequence reserves max_len slots up front
    (§先占好最长的位置)."""
    return Fraction(sum(int(c) for c in context_lens), len(context_lens) * max_len)


def expected_utilisation_uniform(lo: int, hi: int, block_size: int) -> Fraction:
    """E[c] / E[ceil(c/bs) * bs] for c uniform on {lo..hi}: the large-batch
    limit of ``utilisation``."""
    n = hi - lo + 1
    num = sum(range(lo, hi + 1))
    den = sum(blocks_for(c, block_size) * block_size for c in range(lo, hi + 1))
    return Fraction(num, 1) / Fraction(den, 1) * Fraction(n, n)
