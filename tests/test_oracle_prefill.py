"""The prompt-phase oracle (CPU) pinned to things other than itself: torch's
scaled-dot-product attention (fp64) with its causal flag for a prompt without
a prefix, an explicit bottom-right causal mask for a prompt after a cached
prefix, the decode oracle row by row, and planted mistakes that must fail."""

import numpy as np
import pytest
import torch

from oracle.attention import decode_attention, prefill_attention


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _sdpa(q, k, v, scale, mask=None, causal=False):
    """q [n][Hq][d], k/v [c][Hkv][d] -> torch SDPA in fp64, GQA by repeating K/V."""
    G = q.shape[1] // k.shape[1]
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(np.repeat(k, G, axis=1)).permute(1, 0, 2)[None]
    vt = torch.from_numpy(np.repeat(v, G, axis=1)).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=None if mask is None else torch.from_numpy(mask),
        is_causal=causal, scale=scale)
    return o[0].permute(1, 0, 2).numpy()


@pytest.mark.parametrize("n,hq,hkv,d", [(1, 2, 2, 8), (9, 4, 2, 16), (33, 8, 1, 8), (20, 6, 3, 4)])
def test_no_prefix_equals_sdpa_causal(n, hq, hkv, d):
    rng = np.random.default_rng(n + hq)
    q, k, v = _rand(rng, n, hq, d), _rand(rng, n, hkv, d), _rand(rng, n, hkv, d)
    out = prefill_attention(q, k, v, 0.37)
    np.testing.assert_allclose(out, _sdpa(q, k, v, 0.37, causal=True), atol=1e-12)


@pytest.mark.parametrize("c,n", [(10, 1), (10, 4), (50, 50), (64, 17), (100, 3)])
def test_prefix_equals_sdpa_bottom_right_mask(c, n):
    rng = np.random.default_rng(c * 7 + n)
    hq, hkv, d = 4, 2, 8
    q, k, v = _rand(rng, n, hq, d), _rand(rng, c, hkv, d), _rand(rng, c, hkv, d)
    # query t sits at position c - n + t and sees keys 0 .. c - n + t
    mask = np.arange(c)[None, :] <= (c - n + np.arange(n))[:, None]
    out = prefill_attention(q, k, v, 0.25)
    np.testing.assert_allclose(out, _sdpa(q, k, v, 0.25, mask=mask), atol=1e-12)


def test_rows_equal_decode_oracle():
    rng = np.random.default_rng(3)
    c, n, hq, hkv, d = 40, 11, 6, 2, 16
    q, k, v = _rand(rng, n, hq, d), _rand(rng, c, hkv, d), _rand(rng, c, hkv, d)
    out = prefill_attention(q, k, v, 0.5)
    for t in range(n):
        p = c - n + t
        np.testing.assert_allclose(out[t], decode_attention(q[t], k[:p + 1], v[:p + 1], 0.5),
                                   atol=1e-13)


def test_first_prompt_token_sees_only_the_prefix_and_itself():
    rng = np.random.default_rng(4)
    c, n = 12, 5
    q, k, v = _rand(rng, n, 1, 4), _rand(rng, c, 1, 4), _rand(rng, c, 1, 4)
    # changing keys and values after position c - n leaves token 0 unchanged
    k2, v2 = k.copy(), v.copy()
    k2[c - n + 1:] += 5.0
    v2[c - n + 1:] -= 3.0
    a = prefill_attention(q, k, v, 1.0)
    b = prefill_attention(q, k2, v2, 1.0)
    np.testing.assert_array_equal(a[0], b[0])
    assert not np.allclose(a[1:], b[1:])


def test_planted_mistakes_fail():
    rng = np.random.default_rng(5)
    c, n, hq, hkv, d = 30, 8, 4, 2, 8
    q, k, v = _rand(rng, n, hq, d), _rand(rng, c, hkv, d), _rand(rng, c, hkv, d)
    good = prefill_attention(q, k, v, 0.3)
    # a top-left aligned mask (query t sees keys 0..t) ignores the prefix
    top_left = np.arange(c)[None, :] <= np.arange(n)[:, None]
    assert np.max(np.abs(good - _sdpa(q, k, v, 0.3, mask=top_left))) > 1e-2
    # no mask at all
    assert np.max(np.abs(good - _sdpa(q, k, v, 0.3))) > 1e-2
    # strict mask (a token not seeing itself)
    strict = np.arange(c)[None, :] < (c - n + np.arange(n))[:, None]
    assert np.max(np.abs(good - _sdpa(q, k, v, 0.3, mask=strict))) > 1e-2


def test_rejects_bad_shapes():
    with pytest.raises(ValueError):
        prefill_attention(np.zeros((5, 2, 4)), np.zeros((4, 2, 4)), np.zeros((4, 2, 4)), 1.0)
    with pytest.raises(ValueError):
        prefill_attention(np.zeros((2, 3, 4)), np.zeros((4, 2, 4)), np.zeros((4, 2, 4)), 1.0)
