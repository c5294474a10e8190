"""The decode round on contiguous histories.  TEST INFRASTRUCTURE ONLY.

One round of the generation phase ("KV 缓存与分页注意力", §一次写一个词元; the
"KV 缓存" topic page, level 3, the cached generation function): every running
sequence first stores its new token's key and value - into the last slot of
its last block, a fresh block only when that one is full (§块表) - and then
attends over its whole history *including the new token*.  (The exhibit's
animation reads the cache and then drops the new pins; the topic page's
cached function appends first and then attends.  The second is taken: it is
the one that equals full recomputation.)

The oracle keeps, per sequence, the rows it stored, in the representation the
pool holds them (float32 / fp16 / bf16 bit patterns, or FP8-E4M3 codes), and a
``BlockManager`` for the tables.  Attention runs over the contiguous rows,
decoded exactly to float64 (FP8 rows are dequantised as code value * scale).
"""

from __future__ import annotations

from typing import Dict, List, Optional, Sequence

import numpy as np

from .allocator import BlockManager
from .attention import attend_head, decode_attention, prefill_attention
from .numerics import e4m3_decode, e4m3_quantize_for_pool, to_f64

_STORE_NP = {"f32": np.float32, "f16": np.float16, "bf16": np.uint16, "fp8": np.uint8}


class DecodeOracle:
    def __init__(self, num_blocks: int, block_size: int, n_kv_heads: int, head_dim: int,
                 kv_dtype: str, k_scale: float = 1.0, v_scale: float = 1.0,
                 order: Optional[Sequence[int]] = None):
        self.bm = BlockManager(num_blocks, block_size, order)
        self.n_kv_heads = n_kv_heads
        self.head_dim = head_dim
        self.kv_dtype = kv_dtype
        self.k_scale = float(np.float32(k_scale))
        self.v_scale = float(np.float32(v_scale))
        self.k_rows: Dict[int, List[np.ndarray]] = {}
        self.v_rows: Dict[int, List[np.ndarray]] = {}

    # -- storage representation -------------------------------------------
    def stored(self, x: np.ndarray, in_dtype: str, which: str) -> np.ndarray:
        """What the pool holds for input rows ``x`` given in ``in_dtype``
        (float32 / float16 arrays, or bf16 bit patterns)."""
        if self.kv_dtype == "fp8":
            scale = self.k_scale if which == "k" else self.v_scale
            return e4m3_quantize_for_pool(to_f64(x, in_dtype).astype(np.float32), scale)
        if in_dtype != self.kv_dtype:
            raise ValueError("a non-FP8 pool takes rows in its own dtype")
        return np.asarray(x, dtype=_STORE_NP[self.kv_dtype]).copy()

    def dequant(self, rows: np.ndarray, which: str) -> np.ndarray:
        if self.kv_dtype == "fp8":
            scale = self.k_scale if which == "k" else self.v_scale
            return e4m3_decode(rows) * scale
        return to_f64(rows, self.kv_dtype)

    # -- calls ---------------------------------------------------------------
    def admit(self, seq: int, k: np.ndarray, v: np.ndarray, in_dtype: str) -> List[int]:
        """A prompt of n tokens: k, v [n][H_kv][d].  Returns the n slots."""
        slots = self.bm.alloc(seq, k.shape[0])
        ks = self.stored(k, in_dtype, "k")
        vs = self.stored(v, in_dtype, "v")
        self.k_rows[seq] = [ks[t] for t in range(k.shape[0])]
        self.v_rows[seq] = [vs[t] for t in range(v.shape[0])]
        return slots

    def admit_prefix(self, seq: int, tokens, k: np.ndarray, v: np.ndarray, in_dtype: str):
        """A prompt with token ids and all of its rows; with prefix caching on
        the allocator may take over registered blocks for its leading full
        blocks ("KV 缓存与分页注意力" §后来的做法).  The history is the prompt's own
        rows either way.  Returns (slots, n_cached)."""
        slots, n_cached = self.bm.alloc_prefix(seq, tokens)
        ks = self.stored(k, in_dtype, "k")
        vs = self.stored(v, in_dtype, "v")
        self.k_rows[seq] = [ks[t] for t in range(k.shape[0])]
        self.v_rows[seq] = [vs[t] for t in range(v.shape[0])]
        return slots, n_cached

    def fork(self, parent: int, child: int) -> None:
        self.bm.fork(parent, child)
        self.k_rows[child] = list(self.k_rows[parent])
        self.v_rows[child] = list(self.v_rows[parent])

    def free(self, seq: int) -> None:
        self.bm.free_seq(seq)
        del self.k_rows[seq]
        del self.v_rows[seq]

    def swap_out(self, seq: int):
        """"KV 缓存与分页注意力" §放不下的时候: a sequence gives up all of its
        blocks, its keys and values moving to CPU memory.  Returns the stored
        rows ([n][H_kv][d] each) and releases the sequence."""
        rows = self.history(seq) if self.k_rows[seq] else (None, None)
        self.free(seq)
        return rows

    def swap_in(self, seq: int, k_rows: np.ndarray, v_rows: np.ndarray) -> List[int]:
        """The swapped-out rows come back into fresh blocks (an admission of
        the same length); returns the slots."""
        n = 0 if k_rows is None else k_rows.shape[0]
        slots = self.bm.alloc(seq, n)
        self.k_rows[seq] = [k_rows[t] for t in range(n)]
        self.v_rows[seq] = [v_rows[t] for t in range(n)]
        return slots

    def append(self, seqs: Sequence[int], k_new: np.ndarray, v_new: np.ndarray, in_dtype: str):
        """Store one new row per sequence (k_new, v_new [B][H_kv][d]).
        Returns (slots, cow pairs)."""
        slots, pairs = self.bm.append_batch(seqs)
        ks = self.stored(k_new, in_dtype, "k")
        vs = self.stored(v_new, in_dtype, "v")
        for i, s in enumerate(seqs):
            self.k_rows[int(s)].append(ks[i])
            self.v_rows[int(s)].append(vs[i])
        return slots, pairs

    def history(self, seq: int):
        """Stored K and V rows of a sequence, contiguous: [c][H_kv][d]."""
        return np.stack(self.k_rows[seq]), np.stack(self.v_rows[seq])

    def attend(self, seqs: Sequence[int], q: np.ndarray, q_dtype: str, scale: float,
               heads: Optional[Sequence[int]] = None) -> np.ndarray:
        """Attention of each sequence's query over its contiguous history.
        q [B][H_q][d] in q_dtype; returns float64 [B][H_q][d] (or only the listed
        heads, [B][len(heads)][d])."""
        qd = to_f64(q, q_dtype)
        outs = []
        for i, s in enumerate(seqs):
            kh, vh = self.history(int(s))
            kd = self.dequant(kh, "k")
            vd = self.dequant(vh, "v")
            if heads is None:
                outs.append(decode_attention(qd[i], kd, vd, scale))
            else:
                group = qd.shape[1] // self.n_kv_heads
                outs.append(np.stack([
                    attend_head(qd[i][h], kd[:, h // group, :], vd[:, h // group, :], scale)
                    for h in heads]))
        return np.stack(outs)

    def prefill(self, seq: int, q: np.ndarray, q_dtype: str, scale: float) -> np.ndarray:
        """Prompt-phase attention: q [n][H_q][d] are the queries of the last n
        stored tokens of the sequence; returns float64 [n][H_q][d]."""
        kh, vh = self.history(int(seq))
        return prefill_attention(to_f64(q, q_dtype), self.dequant(kh, "k"), self.dequant(vh, "v"),
                                 scale)

    def step(self, seqs: Sequence[int], q: np.ndarray, k_new: np.ndarray, v_new: np.ndarray,
             in_dtype: str, scale: float):
        """Append first, then attend (the new token attends to itself)."""
        slots, pairs = self.append(seqs, k_new, v_new, in_dtype)
        out = self.attend(seqs, q, in_dtype, scale)
        return slots, pairs, out


def gather_rows(pool: np.ndarray, table: Sequence[int], n_tokens: int, block_size: int) -> np.ndarray:
    """Read a sequence's rows out of a pool image [num_blocks][H][bs][d]
    through its block table, in logical token order -> [n][H][d].

    Logical token t lives in block table[t // bs], slot t % bs ("KV 缓存与分页注意力",
    §块表: the kernel fetches keys and values block by block following the
    table; blocks need not be adjacent)."""
    rows = []
    for t in range(n_tokens):
        b = table[t // block_size]
        rows.append(pool[b, :, t % block_size, :])
    if not rows:
        return pool[:0, :, 0, :]
    return np.stack(rows)
