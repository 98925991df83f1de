"""Host checks of the plan restatement the device-planner tests compare with
(tests/plan_ref.py): brute force over the cost line on small batches, so that
the reference itself is pinned to the cost model it states."""

import numpy as np
import pytest

import plan_ref


def brute(seqlens, q_len, max_pages, c_use):
    """Walk the cost line position by position: which cluster holds each page."""
    line = []                       # (sequence, page) or None for overhead units
    for b, L in enumerate(seqlens):
        n = (L + 63) // 64 if q_len <= L <= 64 * max_pages else 0
        if n == 0:
            continue
        line += [None] * plan_ref.SEQ_OVERHEAD + [(b, j) for j in range(n)]
    total = len(line)
    payload = max(plan_ref.MIN_PAYLOAD, -(-total // c_use))
    holders = {}
    for x, item in enumerate(line):
        if item is not None:
            holders.setdefault(item[0], set()).add(x // payload)
    return total, payload, holders


@pytest.mark.parametrize("seed", range(12))
def test_plan_restatement_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 40))
    q_len = int(rng.integers(1, 5))
    max_pages = int(rng.integers(1, 40))
    lens = rng.integers(0, 64 * max_pages + 80, size=B).tolist()   # some invalid (too short or too long)
    c_max = int(rng.integers(1, 75))
    c_use = int(rng.integers(1, c_max + 1))
    p = plan_ref.plan(lens, q_len, 16, max_pages, c_use, c_max)
    total, payload, holders = brute(lens, q_len, max_pages, c_use)
    assert p["hdr"][3] == total and p["hdr"][2] == payload
    assert p["hdr"][1] == (-(-total // payload) if total else 0) <= c_use
    slot = 0
    for b, (start, n, first, splits, s_slot, L) in enumerate(p["seq"]):
        assert L == lens[b]
        held = sorted(holders.get(b, []))
        assert n == (len(held) and (lens[b] + 63) // 64)
        assert splits == len(held)
        if held:
            assert first == held[0] and held == list(range(first, first + splits))
        assert s_slot == slot
        slot += splits if splits > 1 else 0
    assert p["hdr"][4] == slot
    assert p["list"] == [b for b in range(B) if p["seq"][b][3] != 1]
    # each active cluster's first sequence is the first one with a page or overhead unit in its range
    for c in range(c_max):
        fb = p["first_b"][c]
        if c >= p["hdr"][1]:
            assert fb == B
            continue
        x0 = c * payload
        ends = [p["seq"][b][0] + (p["seq"][b][1] + plan_ref.SEQ_OVERHEAD if p["seq"][b][1] else 0) for b in range(B)]
        assert ends[fb] > x0 and all(ends[b] <= x0 for b in range(fb))
