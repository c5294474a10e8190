"""Oracle pin: cached incremental decoding equals full recomputation.

The KV 缓存 topic page (level 3) checks its two generation paths on 27
configurations and 1,080 prefixes and reports a max abs error of 6.7e-16.  The
same check on the oracle's own attend: 27 configurations (layers x dim x seed)
of 40 positions each = 1,080 prefixes.
"""

import itertools

import numpy as np
import pytest

from oracle import toy_transformer as tt


def test_cached_equals_recompute_1080_prefixes():
    worst = 0.0
    prefixes = 0
    for layers, dim, seed in itertools.product((1, 2, 3), (8, 16, 32), (0, 1, 2)):
        w, _, _, sizes = tt.run_both(layers, dim, 40, seed)
        worst = max(worst, w)
        prefixes += len(sizes)
    assert prefixes == 1080
    assert worst < 1e-13


def test_cached_without_self_would_differ():
    # planted mistake: attending before the new key/value is stored makes the
    # cached path disagree with recomputation, so the check above has teeth
    model = tt.make_model(2, 8, 0)
    xs = tt.make_inputs(6, 8, 0)
    cnt = tt.MacCounter()
    cache = tt.Cache(model)
    worst = 0.0
    for t in range(1, 6):
        full = tt.recompute(model, xs[: t + 1], cnt)[-1]
        if t == 1:
            tt.step_cached(model, xs[0], cache, cnt)
        h = xs[t]
        for l in range(model.layers):
            qv = model.wq[l] @ h
            h_new = tt.attend_head(qv, np.stack(cache.k[l]), np.stack(cache.v[l]), 1 / np.sqrt(8))
            cache.k[l].append(model.wk[l] @ h)
            cache.v[l].append(model.wv[l] @ h)
            h = h_new
        worst = max(worst, float(np.max(np.abs(full - h))))
    assert worst > 1e-3
