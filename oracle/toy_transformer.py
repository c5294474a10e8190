"""Cached incremental decoding vs full recomputation.  TEST INFRASTRUCTURE ONLY.

The "KV 缓存" topic page (aiinfact.com), level 3, runs a small attention-only
model (L layers of dimension D, N fixed random input vectors, no vocabulary)
two ways and requires the two to agree:

* without a cache, every prefix is pushed through all layers again; inside a
  layer every position is updated before the next layer starts, and position
  i attends over positions 0..i;
* with a cache, only the new position's key and value are computed per layer,
  appended to that layer's cache, and the new query attends over the cache.

It counts multiply-accumulates (MAC = one multiply plus one add) in two
accounts (level 3 table "账 A / 账 B"):

* account A - the K and V projections only;
* account B - the Q, K and V projections plus the scores and the weighted sum.

Softmax, the 1/sqrt(d) scaling and loop overhead are in neither account.

This module is written from that description; the attention step is
``oracle.attention.attend_head`` with scale 1/sqrt(D).  Counts are accumulated
as the operations run, not from a formula.
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
    wq: List[np.ndarray]
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


def _project(w: np.ndarray, x: np.ndarray, cnt: MacCounter, which: str) -> np.ndarray:
    setattr(cnt, which, getattr(cnt, which) + w.shape[0] * w.shape[1])
    return w @ x


def _attend(q, ks, vs, cnt: MacCounter) -> np.ndarray:
    n, d = ks.shape
    cnt.scores += n * d
    cnt.weighted_sum += n * d
    return attend_head(q, ks, vs, 1.0 / math.sqrt(d))


def recompute(model: ToyModel, inputs: np.ndarray, cnt: MacCounter) -> np.ndarray:
    """Push the whole prefix through every layer; return the last layer's output
    at every position, [n][D]."""
    h = np.array(inputs, dtype=np.float64)
    for l in range(model.layers):
        keys = np.stack([_project(model.wk[l], x, cnt, "k_proj") for x in h])
        vals = np.stack([_project(model.wv[l], x, cnt, "v_proj") for x in h])
        new_h = np.empty_like(h)
        for i, x in enumerate(h):
            qv = _project(model.wq[l], x, cnt, "q_proj")
            new_h[i] = _attend(qv, keys[: i + 1], vals[: i + 1], cnt)
        h = new_h            # the whole layer is updated before the next one
    return h


class Cache:
    def __init__(self, model: ToyModel):
        self.k = [[] for _ in range(model.layers)]
        self.v = [[] for _ in range(model.layers)]

    def elements(self) -> int:
        """How many numbers the cache holds (K and V over all layers)."""
        return sum(sum(x.size for x in rows) for rows in self.k + self.v)


def step_cached(model: ToyModel, x: np.ndarray, cache: Cache, cnt: MacCounter) -> np.ndarray:
    """One new position: per layer, compute and store only its own key and
    value, then attend over the stored ones (itself included)."""
    h = np.asarray(x, dtype=np.float64)
    for l in range(model.layers):
        cache.k[l].append(_project(model.wk[l], h, cnt, "k_proj"))
        cache.v[l].append(_project(model.wv[l], h, cnt, "v_proj"))
        qv = _project(model.wq[l], h, cnt, "q_proj")
        h = _attend(qv, np.stack(cache.k[l]), np.stack(cache.v[l]), cnt)
    return h


def run_both(layers: int, dim: int, n: int, seed: int):
    """Generate n positions both ways.  Returns (max abs difference over all
    prefixes, uncached counter, cached counter, cache element count after each
    position)."""
    model = make_model(layers, dim, seed)
    xs = make_inputs(n, dim, seed)
    c_un = MacCounter()
    c_ca = MacCounter()
    cache = Cache(model)
    worst = 0.0
    sizes = []
    for t in range(n):
        full = recompute(model, xs[: t + 1], c_un)[-1]
        inc = step_cached(model, xs[t], cache, c_ca)
        worst = max(worst, float(np.max(np.abs(full - inc))))
        sizes.append(cache.elements())
    return worst, c_un, c_ca, sizes
