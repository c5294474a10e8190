"""Oracle pins for the number formats (CPU only).

FP8-E4M3 decoding is checked exhaustively over all 256 codes against torch's
float8_e4m3fn (a library routine), and encoding against torch's cast inside the
finite range plus the saturation and tie cases the OCP definition fixes.
"""

import numpy as np
import pytest
import torch

from oracle import numerics as nx


def test_decode_all_codes_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = nx.e4m3_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert set(np.flatnonzero(nan)) == {0x7F, 0xFF}


def test_format_landmarks():
    assert nx.e4m3_decode(np.array([0x7E], np.uint8))[0] == 448.0
    assert nx.e4m3_decode(np.array([0x01], np.uint8))[0] == 2.0 ** -9
    assert nx.e4m3_decode(np.array([0x08], np.uint8))[0] == 2.0 ** -6
    assert nx.e4m3_decode(np.array([0x38], np.uint8))[0] == 1.0
    assert nx.e4m3_decode(np.array([0xB8], np.uint8))[0] == -1.0


def test_encode_matches_torch_in_range():
    g = np.random.default_rng(5)
    x = np.concatenate([
        g.standard_normal(200000) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)
    ]).astype(np.float32)
    x = x[np.abs(x) <= 448.0]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = nx.e4m3_encode(x.astype(np.float64))
    assert np.array_equal(got, ref)


def test_encode_roundtrip_every_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(nx.e4m3_encode(nx.e4m3_decode(codes)), codes)


def test_saturation_and_ties():
    enc = lambda v: int(nx.e4m3_encode(np.array([v]))[0])
    assert enc(448.0) == 0x7E
    assert enc(464.0) == 0x7E          # would round up to 480, which does not exist
    assert enc(1e9) == 0x7E
    assert enc(-1e9) == 0xFE
    assert enc(2.0 ** -10) == 0x00      # tie between 0 and 2^-9: even code
    assert enc(3 * 2.0 ** -10) == 0x02  # tie between codes 1 and 2: even code
    assert enc(1.0 + 1 / 16) == 0x38    # tie between 1.0 (even) and 1.125
    assert enc(1.0 + 3 / 16) == 0x3A    # tie between 1.125 and 1.25 (even)
    assert enc(float("nan")) == 0x7F
    assert enc(-0.0) == 0x80


def test_quantize_for_pool_divides_in_float32():
    x = np.array([1.0, -2.5, 447.9], dtype=np.float32)
    s = np.float32(0.0137)
    got = nx.e4m3_quantize_for_pool(x, float(s))
    want = nx.e4m3_encode((x / s).astype(np.float64))
    assert np.array_equal(got, want)


def test_bf16_and_f16_decode_exact():
    v = np.array([1.0, -2.0, 0.15625, 65504.0], dtype=np.float16)
    assert np.array_equal(nx.f16_to_f64(v), v.astype(np.float64))
    bits = torch.tensor([1.0, -3.5, 1e-20, 3e38], dtype=torch.bfloat16).view(torch.uint16).numpy()
    ref = torch.from_numpy(bits).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(nx.bf16_bits_to_f64(bits), ref)
