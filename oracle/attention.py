"""Decode attention, written as its plain definition.  TEST INFRASTRUCTURE ONLY.

The generation phase ("KV 缓存与分页注意力", §一次写一个词元): each round one new
token computes its own key and value, and then attends over the keys and
values of every earlier token.  PagedAttention (§块表, and "读懂PagedAttention",
§分离逻辑顺序与实际存储位置) reads those keys and values block by block through
the block table; the token order is unchanged.  So the result it reaches is
exactly attention over the sequence's *contiguous* history, and that is what
this module computes:

    s_j   = scale * <q_h, K_{g,j}>          j = 0 .. c-1
    out_h = sum_j softmax(s)_j * V_{g,j}

with g = floor(h / G), G = H_q / H_kv (query heads grouped onto shared KV
heads; "KV 缓存与分页注意力", §后来的做法: Falcon-7B shares one K/V over all heads,
Llama-2-70B puts 64 heads on 8 K/V groups).  The page is silent on which query
heads share a KV head; contiguous groups are taken.  The default scale is
1/sqrt(d) (the "1/sqrt(d) 缩放乘" named on the "KV 缓存" topic page, level 3).

The softmax is the max-subtracted two-pass form, in float64.
"""

from __future__ import annotations

import numpy as np


def softmax(s: np.ndarray) -> np.ndarray:
    """Two-pass softmax of a score vector: subtract the max, exponentiate,
    divide by the sum."""
    s = np.asarray(s, dtype=np.float64)
    m = np.max(s)
    e = np.exp(s - m)
    return e / np.sum(e)


def attend_head(q: np.ndarray, k_hist: np.ndarray, v_hist: np.ndarray, scale: float) -> np.ndarray:
    """One query vector against one head's contiguous history.

    q [d], k_hist [c][d], v_hist [c][d] -> [d] (float64).
    """
    q = np.asarray(q, dtype=np.float64)
    k_hist = np.asarray(k_hist, dtype=np.float64)
    v_hist = np.asarray(v_hist, dtype=np.float64)
    if k_hist.shape[0] == 0:
        raise ValueError("attention over an empty history is undefined")
    s = scale * (k_hist @ q)
    p = softmax(s)
    return p @ v_hist


def decode_attention(q: np.ndarray, k_hist: np.ndarray, v_hist: np.ndarray, scale: float) -> np.ndarray:
    """Decode attention of one sequence.

    q [H_q][d]; k_hist, v_hist [c][H_kv][d] (the sequence's contiguous history,
    the new token included).  Returns out [H_q][d] in float64.
    """
    q = np.asarray(q, dtype=np.float64)
    k_hist = np.asarray(k_hist, dtype=np.float64)
    v_hist = np.asarray(v_hist, dtype=np.float64)
    h_q = q.shape[0]
    h_kv = k_hist.shape[1]
    if h_q % h_kv:
        raise ValueError("n_q_heads must be a multiple of n_kv_heads")
    if k_hist.shape[0] == 0:
        raise ValueError("attention over an empty history is undefined")
    group = h_q // h_kv
    out = np.empty_like(q)
    for g in range(h_kv):
        # the query heads of KV head g, all at once: S = scale * Q K^T [G][c]
        qg = q[g * group:(g + 1) * group]
        s = scale * (qg @ k_hist[:, g, :].T)
        s = s - s.max(axis=1, keepdims=True)
        e = np.exp(s)
        p = e / e.sum(axis=1, keepdims=True)
        out[g * group:(g + 1) * group] = p @ v_hist[:, g, :]
    return out


def attention_weights(q: np.ndarray, k_hist: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * K q) for one head: [c] weights (for the sum-to-one and
    special-case checks)."""
    return softmax(scale * (np.asarray(k_hist, np.float64) @ np.asarray(q, np.float64)))
