"""Oracle pin: cached incremental decoding equals full recomputation.

The KV 缓存 topic page (level 3) checks its two generation paths on 27
configurations and 1,080 prefixes and reports a max abs error of 6.7e-16.  The
same check on the oracle's two independent restatements (masked matrix
attention per layer vs an incremental cache): 27 configurations
(layers x dim x seed) of 40 positions each = 1,080 prefixes.  Two planted
mistakes must break it: attending before the new key and value are stored,
and the one the page itself warns about - updating only the last position of
a layer, so that the next layer reads stale history.
"""

import itertools
import math

import numpy as np

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
    # planted mistake: the new query attends over the cache before its own key
    # and value are stored there
    model = tt.make_model(2, 8, 0)
    xs = tt.make_inputs(6, 8, 0)
    cnt = tt.MacCounter()
    cache = tt.Cache(model, capacity=8)
    tt.step_cached(model, xs[0], cache, cnt)
    worst = 0.0
    for t in range(1, 6):
        full = tt.recompute(model, xs[: t + 1], cnt)[-1]
        h = xs[t]
        for l in range(model.layers):
            q = model.wq[l] @ h
            h_new = tt.attend_head(q, cache.k[l, :t], cache.v[l, :t], 1 / math.sqrt(8))
            cache.k[l, t] = model.wk[l] @ h
            cache.v[l, t] = model.wv[l] @ h
            h = h_new
        cache.length = t + 1
        worst = max(worst, float(np.max(np.abs(full - h))))
    assert worst > 1e-3


def test_stale_history_would_differ():
    # planted mistake: each layer recomputes only the last position and the
    # next layer reads the previous layer's *input* at the earlier positions
    model = tt.make_model(2, 8, 1)
    xs = tt.make_inputs(6, 8, 1)
    cnt = tt.MacCounter()
    full = tt.recompute(model, xs, cnt)[-1]
    h = np.array(xs)
    for l in range(model.layers):
        last = tt._causal_layer(h, model.wq[l], model.wk[l], model.wv[l], cnt)[-1]
        h = np.concatenate([h[:-1], last[None]], axis=0)
    assert float(np.max(np.abs(full - h[-1]))) > 1e-3


def test_matrix_layer_matches_row_by_row_definition():
    # the masked matrix form against the per-row definition of one layer:
    # row i is the single-query attention over keys/values 0..i
    model = tt.make_model(1, 16, 3)
    h = tt.make_inputs(9, 16, 3)
    out = tt._causal_layer(h, model.wq[0], model.wk[0], model.wv[0], tt.MacCounter())
    k = h @ model.wk[0].T
    v = h @ model.wv[0].T
    for i in range(9):
        q = model.wq[0] @ h[i]
        ref = tt.attend_head(q, k[: i + 1], v[: i + 1], 1 / 4.0)
        assert np.max(np.abs(out[i] - ref)) < 1e-14
