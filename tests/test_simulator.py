"""The exhibit's allocation bench (CPU): the reference simulator pinned to a
hand-worked walk and to closed forms, and the library's native simulator
against it, field by field, over seeded request streams of the exhibit's shape
(176 slots, sequences of at most 20 tokens)."""

import json
import os
from fractions import Fraction

import numpy as np
import pytest

import pagedattention_decode_02_b200 as pk
import workloads as W
from oracle.simulator import MAX, ORACLE, POW2, reservation, simulate

GOLD = os.path.join(os.path.dirname(__file__), "golden")
FIELDS = ("rounds", "peak_running", "preemptions", "admitted", "stored_token_rounds",
          "reserved_slot_rounds", "future_slot_rounds", "internal_frag_slot_rounds")
MODES = (1, 2, 4, 8, 16, MAX, POW2, ORACLE)


@pytest.mark.parametrize("native", [False, True])
def test_worked_example(native):
    g = json.load(open(os.path.join(GOLD, "simulator_worked_example.json")))
    reqs = [tuple(r) for r in g["requests"]]
    for mode, want in g["cases"].items():
        if native:
            got, per = pk.pkv_simulate(reqs, g["num_slots"], int(mode), g["max_len"])
            assert got["mean_utilisation"] == pytest.approx(
                want["mean_utilisation"][0] / want["mean_utilisation"][1], abs=1e-12)
        else:
            got = simulate(reqs, g["num_slots"], int(mode), g["max_len"])
            per = got["running_per_round"]
            assert got["mean_utilisation"] == Fraction(*want["mean_utilisation"])
        for f in FIELDS:
            assert got[f] == want[f], (mode, f)
        assert list(per) == want["running_per_round"], mode


def test_reservation_sizes():
    assert [reservation(t, POW2, 20) for t in (1, 2, 3, 4, 5, 9, 16, 17, 20)] == \
        [1, 2, 4, 4, 8, 16, 16, 20, 20]
    assert reservation(7, MAX, 20) == 20 and reservation(7, ORACLE, 20) == 7


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("p,o,a", [(1, 1, 0), (3, 5, 2), (7, 13, 0), (19, 1, 4)])
def test_single_request_closed_form(mode, p, o, a):
    """Alone, a request is admitted on arrival, writes one token a round for o
    rounds and leaves: it holds memory for o+1 rounds with p..p+o tokens."""
    r = simulate([(a, p, o)], W.EXHIBIT_SLOTS, mode, W.EXHIBIT_MAX_LEN)
    assert r["rounds"] == a + o + 1
    assert r["stored_token_rounds"] == (o + 1) * p + o * (o + 1) // 2
    if mode > 0:
        held = sum(-(-(p + k) // mode) * mode for k in range(o + 1))
    else:
        held = (o + 1) * {MAX: 20, POW2: min(20, 1 << (p + o - 1).bit_length()), ORACLE: p + o}[mode]
    assert r["reserved_slot_rounds"] == held
    assert r["preemptions"] == 0 and r["peak_running"] == 1


@pytest.mark.parametrize("seed", range(6))
def test_invariants_and_pins(seed):
    reqs = W.exhibit_requests(60, seed, per_round=3)
    last = max(a + o for a, _, o in reqs)
    for mode in MODES:
        r = simulate(reqs, W.EXHIBIT_SLOTS, mode, W.EXHIBIT_MAX_LEN)
        # every held slot is stored, written later, or never written
        assert (r["stored_token_rounds"] + r["future_slot_rounds"] + r["internal_frag_slot_rounds"]
                == r["reserved_slot_rounds"])
        assert r["rounds"] >= last + 1
        assert r["admitted"] == len(reqs) + r["preemptions"]
        if mode == 1:
            # one-token blocks hold exactly the tokens written
            assert r["mean_utilisation"] == 1 and r["internal_frag_slot_rounds"] == 0
            assert r["future_slot_rounds"] == 0
        if mode > 0:
            # paged: at most block_size - 1 unwritten slots per running request
            assert r["future_slot_rounds"] + r["internal_frag_slot_rounds"] <= \
                (mode - 1) * sum(r["running_per_round"])
        else:
            assert r["preemptions"] == 0
        if mode == MAX:
            # 176 slots hold floor(176 / 20) = 8 full-length reservations; with a
            # queue that never drains early, exactly 8 run at the peak
            assert r["peak_running"] == W.EXHIBIT_SLOTS // W.EXHIBIT_MAX_LEN
        if mode == ORACLE:
            assert r["internal_frag_slot_rounds"] == 0


def test_ample_memory_never_waits():
    """With room for every request at once, each leaves in the round it
    writes its last token: rounds = max(arrival + output) + 1."""
    reqs = W.exhibit_requests(40, 3, per_round=2)
    last = max(a + o for a, _, o in reqs)
    for mode in MODES:
        r = simulate(reqs, 40 * 32, mode if mode != 16 else 16, W.EXHIBIT_MAX_LEN)
        assert r["rounds"] == last + 1 and r["preemptions"] == 0
        assert r["admitted"] == len(reqs)


def test_smaller_blocks_waste_less():
    """The exhibit's point: the bigger the block, the more of the last block
    stays empty; a contiguous max-length reservation wastes the most."""
    reqs = W.exhibit_requests(80, 11, per_round=1)
    util = {m: float(simulate(reqs, W.EXHIBIT_SLOTS, m, W.EXHIBIT_MAX_LEN)["mean_utilisation"])
            for m in MODES}
    assert util[1] == 1.0
    assert util[1] >= util[2] >= util[4] >= util[8] >= util[16]
    assert util[ORACLE] >= util[POW2] >= util[MAX]
    assert util[4] > util[MAX]


@pytest.mark.parametrize("seed", range(12))
@pytest.mark.parametrize("per_round", [1, 2, 4])
def test_native_matches_reference(seed, per_round):
    reqs = W.exhibit_requests(24 + 8 * seed, seed, per_round)
    for mode in MODES:
        a, per = pk.pkv_simulate(reqs, W.EXHIBIT_SLOTS, mode, W.EXHIBIT_MAX_LEN)
        b = simulate(reqs, W.EXHIBIT_SLOTS, mode, W.EXHIBIT_MAX_LEN)
        for f in FIELDS:
            assert a[f] == b[f], (mode, f)
        assert a["mean_utilisation"] == pytest.approx(float(b["mean_utilisation"]), abs=1e-12)
        assert per.tolist() == b["running_per_round"]


def test_native_preempts_under_pressure():
    # many long requests at once on a small pool forces preemption
    reqs = [(0, 8, 12)] * 12
    a, _ = pk.pkv_simulate(reqs, 64, 4, 20)
    b = simulate(reqs, 64, 4, 20)
    assert a["preemptions"] > 0
    for f in FIELDS:
        assert a[f] == b[f], f


def test_native_rejects_bad_input():
    with pytest.raises(pk.PagedKVError):
        pk.pkv_simulate([(0, 0, 3)], 16, 4, 20)            # empty prompt
    with pytest.raises(pk.PagedKVError):
        pk.pkv_simulate([(0, 15, 10)], 16, 4, 20)          # longer than max_len
    with pytest.raises(pk.PagedKVError):
        pk.pkv_simulate([(1, 2, 2), (0, 2, 2)], 16, 4, 20)  # arrivals out of order
    with pytest.raises(pk.PagedKVError):
        pk.pkv_simulate([(0, 2, 2)], 18, 4, 20)            # slots not whole blocks
    with pytest.raises(pk.PagedKVError):
        pk.pkv_simulate([(0, 2, 2)], 16, -3, 20)           # unknown mode
    with pytest.raises(pk.PagedKVError):
        pk.pkv_simulate([(0, 2, 30)], 16, 4, 40, max_rounds=5)   # too few rounds
    r, per = pk.pkv_simulate([], 16, 4, 20)
    assert r["rounds"] == 0 and len(per) == 0
