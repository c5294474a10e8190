"""Oracle pins for decode attention (CPU only).

Checked against what the mathematics fixes (special cases with analytic
outputs), against library routines (scipy's softmax, torch's fp64
scaled_dot_product_attention) and against the paging invariant: reading the
history through any block table and any physical permutation gives the
contiguous history, so attention over it is unchanged.
"""

import math

import numpy as np
import pytest
import scipy.special
import torch

from oracle.attention import attend_head, attention_weights, decode_attention, softmax
from oracle.engine import DecodeOracle, gather_rows

rng = np.random.default_rng(1234)


def test_single_token_returns_its_value():
    for d in (1, 32, 128):
        q = rng.standard_normal(d)
        k = rng.standard_normal((1, d))
        v = rng.standard_normal((1, d))
        assert np.array_equal(attend_head(q, k, v, 0.3), v[0])


def test_equal_keys_give_mean_of_values():
    d, c = 16, 37
    k = np.tile(rng.standard_normal(d), (c, 1))
    v = rng.standard_normal((c, d))
    out = attend_head(rng.standard_normal(d), k, v, 1 / math.sqrt(d))
    assert np.allclose(out, v.mean(axis=0), atol=1e-14, rtol=0)


def test_zero_query_gives_mean_of_values():
    d, c = 8, 50
    out = attend_head(np.zeros(d), rng.standard_normal((c, d)), v := rng.standard_normal((c, d)), 1.0)
    assert np.allclose(out, v.mean(axis=0), atol=1e-14, rtol=0)


def test_dominant_key_selects_its_value():
    d, c = 32, 20
    q = rng.standard_normal(d)
    k = rng.standard_normal((c, d))
    k[7] = 1e3 * q / np.linalg.norm(q)
    v = rng.standard_normal((c, d))
    out = attend_head(q, k, v, 1 / math.sqrt(d))
    assert np.allclose(out, v[7], atol=1e-12, rtol=0)


def test_weights_are_a_distribution_and_match_scipy():
    for c in (1, 2, 17, 300):
        q = rng.standard_normal(64)
        k = rng.standard_normal((c, 64)) * 3
        w = attention_weights(q, k, 0.125)
        assert np.all(w >= 0)
        assert abs(w.sum() - 1) < 1e-14
        ref = scipy.special.softmax(0.125 * (k @ q))
        assert np.allclose(w, ref, atol=1e-15, rtol=1e-13)


def test_softmax_shift_invariance_and_large_scores():
    s = rng.standard_normal(40) * 50
    assert np.allclose(softmax(s), softmax(s + 1e4), atol=1e-15)
    assert np.all(np.isfinite(softmax(s * 1e3)))


@pytest.mark.parametrize("h_q,h_kv", [(1, 1), (4, 4), (8, 2), (71, 1), (64, 8)])
def test_matches_torch_sdpa_fp64(h_q, h_kv):
    d, c = 64, 45
    q = rng.standard_normal((h_q, d))
    k = rng.standard_normal((c, h_kv, d))
    v = rng.standard_normal((c, h_kv, d))
    scale = 1 / math.sqrt(d)
    out = decode_attention(q, k, v, scale)
    g = h_q // h_kv
    # library: torch SDPA on CPU in fp64, heads expanded by repeat_interleave
    kt = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(g, dim=0)    # [H_q][c][d]
    vt = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(g, dim=0)
    qt = torch.from_numpy(q)[:, None, :]                                      # [H_q][1][d]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)[:, 0, :].numpy()
    assert np.allclose(out, ref, atol=1e-13, rtol=0)


def test_gqa_head_map_is_contiguous_groups():
    # each KV head g has constant keys, so query head h gets the mean of head
    # floor(h / G)'s values
    h_q, h_kv, d, c = 12, 3, 4, 9
    k = np.ones((c, h_kv, d))
    v = rng.standard_normal((c, h_kv, d))
    out = decode_attention(rng.standard_normal((h_q, d)), k, v, 1.0)
    for h in range(h_q):
        assert np.allclose(out[h], v[:, h // 4, :].mean(axis=0), atol=1e-14)


def test_transposed_or_wrong_group_would_fail():
    # planted mistakes a plausible bug could make; each must change the result
    h_q, h_kv, d, c = 8, 2, 16, 30
    q = rng.standard_normal((h_q, d))
    k = rng.standard_normal((c, h_kv, d))
    v = rng.standard_normal((c, h_kv, d))
    good = decode_attention(q, k, v, 0.25)
    swapped = decode_attention(q, k[:, ::-1], v[:, ::-1], 0.25)
    assert np.max(np.abs(good - swapped)) > 1e-3
    no_scale = decode_attention(q, k, v, 1.0)
    assert np.max(np.abs(good - no_scale)) > 1e-3


@pytest.mark.parametrize("bs", [1, 2, 3, 4, 7, 16, 64])
def test_paged_equals_contiguous_any_block_size_and_permutation(bs):
    h_kv, d = 2, 8
    lens = [1, bs, bs + 1, 3 * bs, 5 * bs - 1, 40]
    need = sum(-(-n // bs) for n in lens)
    order = rng.permutation(need + 3)
    orc = DecodeOracle(need + 3, bs, h_kv, d, "f32", order=order)
    pool = np.full((need + 3, h_kv, bs, d), np.nan, dtype=np.float32)
    hists = {}
    for s, n in enumerate(lens):
        k = rng.standard_normal((n, h_kv, d)).astype(np.float32)
        v = rng.standard_normal((n, h_kv, d)).astype(np.float32)
        slots = orc.admit(s, k, v, "f32")
        for t, sl in enumerate(slots):               # scatter rows by slot
            pool[sl // bs, :, sl % bs, :] = k[t]
        hists[s] = k
    tables, lens_out, _ = orc.bm.export(range(len(lens)), 64)
    for s, n in enumerate(lens):
        got = gather_rows(pool, tables[s], lens_out[s], bs)
        assert np.array_equal(got, hists[s])
        kh, _ = orc.history(s)
        assert np.array_equal(kh, hists[s])
    # attention over the gathered rows is bit-identical to the contiguous one
    q = rng.standard_normal((h_kv, d))
    g = gather_rows(pool, tables[4], lens_out[4], bs).astype(np.float64)
    assert np.array_equal(decode_attention(q, g, g, 0.3),
                          decode_attention(q, hists[4].astype(np.float64), hists[4].astype(np.float64), 0.3))
