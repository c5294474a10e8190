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


def prefill_attention(q: np.ndarray, k_hist: np.ndarray, v_hist: np.ndarray,
                      scale: float) -> np.ndarray:
    """Prompt-phase attention of one sequence over its paged cache.

    "KV 缓存与分页注意力", §一次写一个词元: the prompt phase computes the whole
    prompt at once.  Its n tokens are the last n of the history (their keys and
    values already stored, after any cached prefix: §后来的做法, or after a
    preemption whose prompt and written tokens are recomputed as one new
    prompt: §放不下的时候).  Token t of them, at position c - n + t, attends to
    positions 0 .. c - n + t, itself included (causal):

        out[t][h] = sum_{j <= c-n+t} softmax_j(scale * <q[t][h], K_{g,j}>) V_{g,j}

    q [n][H_q][d]; k_hist, v_hist [c][H_kv][d] with c >= n.  Returns
    [n][H_q][d] float64.
    """
    q = np.asarray(q, dtype=np.float64)
    k_hist = np.asarray(k_hist, dtype=np.float64)
    v_hist = np.asarray(v_hist, dtype=np.float64)
    n, h_q, _ = q.shape
    c, h_kv, _ = k_hist.shape
    if h_q % h_kv:
        raise ValueError("n_q_heads must be a multiple of n_kv_heads")
    if n < 1 or c < n:
        raise ValueError("need 1 <= n <= c")
    group = h_q // h_kv
    pos = np.arange(c - n, c)                          # positions of the n queries
    visible = np.arange(c)[None, :] <= pos[:, None]    # [n][c] causal mask
    out = np.empty_like(q)
    for h in range(h_q):
        g = h // group
        s = scale * (q[:, h, :] @ k_hist[:, g, :].T)    # [n][c]
        s = np.where(visible, s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        e = np.exp(s)
        out[:, h, :] = (e / e.sum(axis=1, keepdims=True)) @ v_hist[:, g, :]
    return out
