"""The exhibit's allocation bench, restated.  TEST INFRASTRUCTURE ONLY.

"KV 缓存与分页注意力" §实验台: sequences arrive one after another, are written
and leave; those that do not fit wait; block size 1, 2, 4, 8 or 16 tokens, or
"max" (every sequence takes a whole row of the maximum length up front,
§先占好最长的位置).  Readouts: the most sequences writing at once, the share of
the reserved memory holding tokens on average, and the rounds it took.  The
paper's other two Orca reservations (§三种浪费) are modes too: the next power
of two of a sequence's final length (at most twice what it needs), and
exactly its final length (known in advance only in a thought experiment).
Held memory splits into slots written later (reservation) and slots never
written (internal fragmentation).

Rules where the page is silent (the same readings as the library's bench):
each round (1) admits waiting requests in arrival order while the head fits,
(2) lets every request admitted in an earlier round write one token - a paged
request that finds no block makes the most recently admitted running request
give up all of its blocks (§放不下的时候), and that request rejoins the head of
the queue with everything it wrote as its new prompt - and (3) lets finished
requests leave.  Readouts are taken after (2).  A contiguous reservation is
placed at the first run of free slots long enough.
"""

from __future__ import annotations

from collections import deque
from fractions import Fraction
from typing import List, Sequence, Tuple

from .allocator import AllocError, BlockManager


MAX, POW2, ORACLE = 0, -1, -2


def reservation(total: int, mode: int, max_len: int) -> int:
    """Slots a contiguous reservation takes for a sequence of final length total."""
    if mode == MAX:
        return max_len
    if mode == ORACLE:
        return total
    if mode == POW2:
        return min(max_len, 1 << (total - 1).bit_length())
    raise ValueError(mode)


def simulate(requests: Sequence[Tuple[int, int, int]], num_slots: int, block_size: int,
             max_len: int, max_rounds: int = 10000) -> dict:
    """requests: (arrival round, prompt tokens, output tokens), arrivals
    non-decreasing.  block_size > 0 pages; MAX, POW2 or ORACLE reserve."""
    paged = block_size > 0
    bm = BlockManager(num_slots // block_size, block_size) if paged else None
    used = [False] * num_slots
    queue: deque = deque()
    arriving = list(range(len(requests)))
    running: List[dict] = []
    order = 0
    out = {"rounds": 0, "peak_running": 0, "preemptions": 0, "admitted": 0,
           "stored_token_rounds": 0, "reserved_slot_rounds": 0, "future_slot_rounds": 0,
           "internal_frag_slot_rounds": 0}
    ratios = []
    per_round = []
    finished = 0
    r = 0
    while finished < len(requests):
        if r >= max_rounds:
            raise RuntimeError("did not finish")
        while arriving and requests[arriving[0]][0] <= r:
            queue.append((arriving.pop(0), 0))
        # (1) admission, head first
        while queue:
            rid, done = queue[0]
            prompt = requests[rid][1] + done
            entry = {"id": rid, "written": prompt, "total": requests[rid][1] + requests[rid][2],
                     "round": r, "order": order, "start": None, "held": None}
            if paged:
                try:
                    bm.alloc(rid, prompt)
                except AllocError:
                    break
            else:
                want = reservation(entry["total"], block_size, max_len)
                start = next((s for s in range(num_slots - want + 1)
                              if not any(used[s:s + want])), None)
                if start is None:
                    break
                used[start:start + want] = [True] * want
                entry["start"], entry["held"] = start, want
            order += 1
            out["admitted"] += 1
            running.append(entry)
            queue.popleft()
        # (2) one token each for requests admitted earlier
        i = 0
        while i < len(running):
            e = running[i]
            if e["round"] == r or e["written"] >= e["total"]:
                i += 1
                continue
            gone = False
            while paged:
                try:
                    bm.append(e["id"])
                    break
                except AllocError:
                    victim = max(running, key=lambda x: x["order"])
                    bm.free_seq(victim["id"])
                    queue.appendleft((victim["id"], victim["written"] - requests[victim["id"]][1]))
                    out["preemptions"] += 1
                    vi = running.index(victim)
                    running.pop(vi)
                    if victim is e:
                        gone = True
                        break
                    if vi < i:
                        i -= 1
            if gone:
                continue
            e["written"] += 1
            i += 1
        # readouts
        stored = reserved = 0
        for e in running:
            held = -(-e["written"] // block_size) * block_size if paged else e["held"]
            will = min(held, e["total"])
            stored += e["written"]
            reserved += held
            out["future_slot_rounds"] += will - e["written"]
            out["internal_frag_slot_rounds"] += held - will
        out["peak_running"] = max(out["peak_running"], len(running))
        out["stored_token_rounds"] += stored
        out["reserved_slot_rounds"] += reserved
        if reserved:
            ratios.append(Fraction(stored, reserved))
        per_round.append(len(running))
        # (3) departures
        for e in [x for x in running if x["written"] >= x["total"]]:
            if paged:
                bm.free_seq(e["id"])
            else:
                used[e["start"]:e["start"] + e["held"]] = [False] * e["held"]
            running.remove(e)
            finished += 1
        r += 1
    out["rounds"] = r
    out["mean_utilisation"] = (sum(ratios) / len(ratios)) if ratios else Fraction(0)
    out["running_per_round"] = per_round
    return out
