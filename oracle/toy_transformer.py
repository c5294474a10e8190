"""Cached incremental decoding vs full recomputation.  TEST INFRASTRUCTURE ONLY.

What the "KV 缓存" topic page (aiinfact.com), level 3, fixes about its small
attention-only model (L layers of dimension D, N fixed random input vectors,
no vocabulary), restated from the mathematics rather than from its script:

* a layer maps the sequence of vectors h_0 .. h_{n-1} to
  out_i = sum_{j <= i} softmax_j(<q_i, k_j> / sqrt(D)) v_j with q = Wq h,
  k = Wk h, v = Wv h - causal self-attention, each position sees itself and
  everything before it;
* layers compose: layer l + 1 reads the outputs of layer l at *every*
  position (the page warns that updating only the last position gives a
  different computation);
* generation without a cache recomputes the whole prefix through all layers
  for every new position; with a cache only the new position's key and value
  are computed per layer and the earlier ones are read back.

Written here as two independent restatements:

* ``recompute`` - per layer one masked matrix attention over the whole prefix
  (Q, K, V as n x D matrices, scores Q K^T / sqrt(D) with the upper triangle
  masked, a row softmax, then P V);
* ``step_cached`` - one position at a time into a preallocated cache
  ``[L][capacity][D]`` with a length counter; the three projections of the
  new position are one stacked [3D x D] product; its query attends over rows
  0 .. t of the layer's cache through ``oracle.attention.attend_head``.

Multiply-accumulates (one multiply plus one add) are counted in the page's
two accounts (level 3 table "账 A / 账 B"): account A - the K and V
projections; account B - the Q, K and V projections plus the scores and the
weighted sum.  Softmax, the 1/sqrt(D) scaling and loop overhead are in
neither.  The counts come from the shapes of the products as they run; a
causal score or weighted-sum term is counted only for the (i, j <= i) pairs,
the ones a causal computation evaluates.
"""

from __future__ import annotations

import dataclasses
import math
from typing import List

import numpy as np

from .attention import attend_head


@dataclasses.dataclass
class MacCounter:
    q_proj: int = 0
    k_proj: int = 0
    v_proj: int = 0
    scores: int = 0
    weighted_sum: int = 0

    @property
    def account_a(self) -> int:
        return self.k_proj + self.v_proj

    @property
    def account_b(self) -> int:
        return self.q_proj + self.k_proj + self.v_proj + self.scores + self.weighted_sum


@dataclasses.dataclass
class ToyModel:
    wq: List[np.ndarray]      # per layer [D][D]: q = wq @ h
    wk: List[np.ndarray]
    wv: List[np.ndarray]

    @property
    def layers(self) -> int:
        return len(self.wq)

    @property
    def dim(self) -> int:
        return self.wq[0].shape[0]


def make_model(layers: int, dim: int, seed: int) -> ToyModel:
    g = np.random.default_rng([seed, 77])
    s = 1.0 / math.sqrt(dim)
    mk = lambda: [g.standard_normal((dim, dim)) * s for _ in range(layers)]
    return ToyModel(mk(), mk(), mk())


def make_inputs(n: int, dim: int, seed: int) -> np.ndarray:
    return np.random.default_rng([seed, 78]).standard_normal((n, dim))


def _matmul(a: np.ndarray, b: np.ndarray) -> tuple:
    """a @ b and its multiply-accumulate count (rows x inner x columns)."""
    m, k = a.shape
    k2, n = b.shape
    assert k == k2
    return a @ b, m * k * n


def _causal_layer(h: np.ndarray, wq, wk, wv, cnt: MacCounter) -> np.ndarray:
    """One layer over a whole prefix h [n][D] as masked matrix attention."""
    n, dim = h.shape
    q, c = _matmul(h, wq.T)
    cnt.q_proj += c
    k, c = _matmul(h, wk.T)
    cnt.k_proj += c
    v, c = _matmul(h, wv.T)
    cnt.v_proj += c
    visible = np.tril(np.ones((n, n), dtype=bool))       # key j visible to query i iff j <= i
    pairs = int(visible.sum())
    s = (q @ k.T) / math.sqrt(dim)
    cnt.scores += pairs * dim
    s = np.where(visible, s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    w = np.exp(s)
    p = w / w.sum(axis=1, keepdims=True)
    cnt.weighted_sum += pairs * dim
    return p @ v


def recompute(model: ToyModel, inputs: np.ndarray, cnt: MacCounter) -> np.ndarray:
    """Push the whole prefix through every layer; return the last layer's output
    at every position, [n][D]."""
    h = np.array(inputs, dtype=np.float64)
    for l in range(model.layers):
        h = _causal_layer(h, model.wq[l], model.wk[l], model.wv[l], cnt)
    return h


class Cache:
    """Keys and values of every generated position, per layer, in preallocated
    arrays [layers][capacity][D]; rows 0 .. length-1 are filled."""

    def __init__(self, model: ToyModel, capacity: int = 64):
        self.k = np.zeros((model.layers, capacity, model.dim))
        self.v = np.zeros((model.layers, capacity, model.dim))
        self.length = 0

    def elements(self) -> int:
        """How many numbers the cache holds (K and V over all layers)."""
        return 2 * self.k.shape[0] * self.length * self.k.shape[2]


def step_cached(model: ToyModel, x: np.ndarray, cache: Cache, cnt: MacCounter) -> np.ndarray:
    """Generate one new position t = cache.length: per layer compute only its
    own query, key and value, store the key and value at row t, then attend
    over rows 0..t (itself included).  Returns the last layer's output."""
    t = cache.length
    if t >= cache.k.shape[1]:
        raise ValueError("cache capacity exceeded")
    dim = model.dim
    h = np.asarray(x, dtype=np.float64)
    for l in range(model.layers):
        w_qkv = np.concatenate([model.wq[l], model.wk[l], model.wv[l]], axis=0)  # [3D][D]
        qkv, _ = _matmul(w_qkv, h[:, None])
        cnt.q_proj += dim * dim
        cnt.k_proj += dim * dim
        cnt.v_proj += dim * dim
        q, k, v = qkv[:dim, 0], qkv[dim:2 * dim, 0], qkv[2 * dim:, 0]
        cache.k[l, t] = k
        cache.v[l, t] = v
        cnt.scores += (t + 1) * dim
        cnt.weighted_sum += (t + 1) * dim
        h = attend_head(q, cache.k[l, : t + 1], cache.v[l, : t + 1], 1.0 / math.sqrt(dim))
    cache.length = t + 1
    return h


def run_both(layers: int, dim: int, n: int, seed: int):
    """Generate n positions both ways.  Returns (max abs difference over all
    prefixes, uncached counter, cached counter, cache element count after each
    position)."""
    model = make_model(layers, dim, seed)
    xs = make_inputs(n, dim, seed)
    c_un = MacCounter()
    c_ca = MacCounter()
    cache = Cache(model, capacity=n)
    worst = 0.0
    sizes = []
    for t in range(n):
        full = recompute(model, xs[: t + 1], c_un)[-1]
        inc = step_cached(model, xs[t], cache, c_ca)
        worst = max(worst, float(np.max(np.abs(full - inc))))
        sizes.append(cache.elements())
    return worst, c_un, c_ca, sizes
