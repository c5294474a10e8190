"""Oracle pins: closed forms and printed values from the pages (CPU only)."""

import json
import os
from fractions import Fraction

import pytest

from oracle import closed_forms as cf
from oracle import toy_transformer as tt

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


@pytest.mark.parametrize("row", _gold("closed_forms.json")["per_token_bytes"], ids=lambda r: r["model"])
def test_per_token_bytes(row):
    got = cf.kv_bytes_per_token(row["layers"], row["n_kv_heads"], row["head_dim"], row["bytes_per_elem"])
    assert got == row["expected"]


def test_printed_units():
    g = _gold("closed_forms.json")
    assert 819200 / 1024 == 800.0                       # "800 KB", binary
    assert 327680 == 320 * 1024 and 8192 == 8 * 1024      # "320 KB", "8 KB"
    r = g["opt13b_ratio_llama2_70b"]
    assert Fraction(327680, 819200) == Fraction(r["numerator"], r["denominator"])
    # one 2,048-token OPT-13B sequence: "up to 1.6 GB"
    seq = g["opt13b_max_sequence"]
    b = cf.kv_cache_bytes(1, 40, seq["tokens"], 40, 128, 2)
    assert b == 819200 * 2048
    assert round(b / 2**30, 1) == seq["approx_gb"]


def test_a100_pool_capacity():
    g = _gold("closed_forms.json")["a100_pool"]
    space = g["kv_space_gib"] * 2**30
    tok = cf.tokens_that_fit(space, 819200)
    assert abs(tok - g["approx_tokens"]) < 50            # "about 15,700"
    assert tok == 15728
    assert cf.max_length_sequences_that_fit(space, 819200, g["max_len"]) == g["max_len_sequences"]


def test_exhibit_machine_slots():
    g = _gold("closed_forms.json")["exhibit_machine"]
    assert g["blocks"] * g["block_size"] == g["slots"]
    # "max" reservation: each sequence takes a whole row of 20 slots
    assert g["slots"] // g["max_seq_tokens"] == 8


def test_waste_below_one_block():
    # section 块表: a sequence wastes at most the unfilled part of its last block
    for bs in (1, 2, 4, 8, 16, 32, 64):
        for c in range(1, 300):
            waste = cf.blocks_for(c, bs) * bs - c
            assert 0 <= waste <= bs - 1


@pytest.mark.parametrize("bs", [1, 2, 4, 8, 16, 32, 64])
def test_expected_utilisation_closed_form(bs):
    # c uniform on {2..2049}: 2048 values, a whole number of residue cycles for
    # every bs <= 64, so the mean waste is (bs - 1) / 2 exactly
    got = cf.expected_utilisation_uniform(2, 2049, bs)
    mean_c = Fraction(2 + 2049, 2)
    assert got == mean_c / (mean_c + Fraction(bs - 1, 2))


def test_utilisation_small_examples():
    assert cf.utilisation([4, 4], 4) == 1
    assert cf.utilisation([5], 4) == Fraction(5, 8)
    assert cf.utilisation([1, 2, 3], 1) == 1
    assert cf.max_reservation_utilisation([10, 10], 20) == Fraction(1, 2)


def test_cache_size_formula_matches_toy():
    # level 1 formula with B=1, L=2, H_kv*d = 32, N positions and "one number"
    # per element gives the level 3 cache column
    g = _gold("kv_cache_topic_counts.json")
    for pos, n in g["cache_elements"].items():
        if pos.isdigit():
            assert cf.kv_cache_bytes(1, 2, int(pos), 1, 32, 1) == n


def test_mac_accounts_and_cache_counts():
    g = _gold("kv_cache_topic_counts.json")
    c = g["config"]
    worst, un, ca, sizes = tt.run_both(c["layers"], c["dim"], c["positions"], seed=0)
    assert un.account_b == g["account_b"]["uncached"]
    assert ca.account_b == g["account_b"]["cached"]
    assert un.account_a == g["account_a"]["uncached"]
    assert ca.account_a == g["account_a"]["cached"]
    n = c["positions"]
    assert Fraction(ca.account_a, un.account_a) == Fraction(2, n + 1)
    assert round(100 * ca.account_b / un.account_b, 3) == 5.389
    for pos, want in g["cache_elements"].items():
        if pos.isdigit():
            assert sizes[int(pos) - 1] == want
    assert sizes[0] == g["cache_elements"]["per_position"]
    assert worst < 1e-13
