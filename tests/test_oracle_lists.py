"""Pins for the oracle's frame sets (no GPU, no library).

What pins what:
* a hand-derived worked example (tests/golden/worked_example_T8_C4_W2.txt) fixes
  the tie-breaks (even-W centring, right-first extension, floor stride);
* brute force over every small (T, C, W, step) checks the properties the pages
  state: |A(t)| = min(C, T); anchors and the initial window are inside A(t);
  the non-anchor frames form one interval; G anchors at every step; the anchor
  set moves by one frame per step modulo T; every frame is an anchor once or
  twice within T_per steps, exactly G*T_per - T frames twice;
* closed forms: C >= T is every frame; G = 0 is a plain clamped sliding window.
* planted mistakes (monkeypatched into the oracle, CPU only) must fail a pin.
"""

import os
import itertools

import pytest

from oracle import lists as OL

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example_T8_C4_W2.txt")


def read_golden():
    rows = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, frames = line.split(":")
            s, t = (int(x) for x in head.split())
            rows[(s, t)] = [int(x) for x in frames.split()]
    return rows


def test_worked_example_matches():
    gold = read_golden()
    assert len(gold) == 24
    for (s, t), frames in gold.items():
        assert OL.frame_set(t, 8, 4, 2, s) == frames, (s, t)


def check_invariants(T, C, W, s):
    L = min(C, T)
    lists = OL.frame_lists(T, C, W, s)
    assert len(lists) == T
    if C >= T:
        for row in lists:
            assert row == list(range(T))
        return
    G = set(OL.anchors(T, C, W, s))
    assert len(G) == C - W
    for t, row in enumerate(lists):
        assert len(row) == L
        assert row == sorted(set(row)), "strictly ascending, no duplicates"
        assert all(0 <= f < T for f in row)
        A = set(row)
        assert G <= A
        lo, hi = OL.window(t, T, W)
        assert hi - lo + 1 == W and 0 <= lo and hi < T and lo <= t <= hi
        assert set(range(lo, hi + 1)) <= A
        # non-anchor frames plus the window span one gap-free interval
        span = (A - G) | set(range(lo, hi + 1))
        a, b = min(span), max(span)
        assert set(range(a, b + 1)) <= A


def small_cases(maxT):
    for T in range(1, maxT + 1):
        for C in range(1, T + 2):
            for W in range(1, C + 1):
                yield T, C, W


def test_invariants_brute_force():
    n = 0
    for T, C, W in small_cases(13):
        for s in range(0, 2 * T + 1):
            check_invariants(T, C, W, s)
            n += 1
    assert n > 5000


def test_rotation_by_one_frame_per_step():
    for T, C, W in small_cases(13):
        if C >= T or C == W:
            continue
        for s in range(0, 2 * T):
            a = OL.anchors(T, C, W, s)
            b = OL.anchors(T, C, W, s + 1)
            assert sorted((f + 1) % T for f in a) == b
            assert len(a) == C - W


def test_coverage_once_or_twice():
    for T, C, W in small_cases(16):
        if C >= T or C == W:
            continue
        G = C - W
        Tper = OL.anchor_period(T, C, W)
        for first in range(0, T):
            counts = OL.anchor_coverage(T, C, W, first)
            assert min(counts) >= 1 and max(counts) <= 2
            assert sum(1 for c in counts if c == 2) == G * Tper - T
            if T % G == 0:
                assert max(counts) == 1  # exactly once when the stride divides T


def test_pure_window_closed_form():
    # G = 0 (W = C < T): a sliding window of C frames, clamped at the ends.
    for T in range(2, 15):
        for C in range(1, T):
            for t in range(T):
                lo = min(max(t - C // 2, 0), T - C)
                assert OL.frame_set(t, T, C, C, 3) == list(range(lo, lo + C))


def test_dense_when_budget_covers_video():
    for T in range(1, 12):
        for C in range(T, T + 3):
            for W in (1, C):
                assert OL.frame_lists(T, C, W, 5) == [list(range(T))] * T


@pytest.mark.parametrize("T,C,W,G,Tper,doubles", [
    (121, 21, 9, 12, 11, 11),   # Wan-1.3B / Wan-14B at 6x horizon
    (49, 33, 13, 20, 3, 11),    # HunyuanVideo-1.5 at 1.5x horizon
    (8, 4, 2, 2, 4, 0),         # tiny case
])
def test_workload_anchor_figures(T, C, W, G, Tper, doubles):
    assert OL.anchor_count(T, C, W) == G
    assert OL.anchor_period(T, C, W) == Tper
    for s in range(50):
        assert len(OL.anchors(T, C, W, s)) == G
        check_invariants(T, C, W, s)
    counts = OL.anchor_coverage(T, C, W, 0)
    assert sum(1 for c in counts if c == 2) == doubles


def test_bad_args():
    for args in [(0, 4, 2, 0), (8, 0, 1, 0), (8, 4, 0, 0), (8, 4, 5, 0), (8, 4, 2, -1)]:
        with pytest.raises(ValueError):
            OL.frame_lists(*args)


# ----------------------------------------------------------------------------
# Planted mistakes: each plausible error in the oracle must fail some pin above.
# ----------------------------------------------------------------------------

def test_mistake_integer_stride_is_caught(monkeypatch):
    # anchors at the integer stride ceil(T/G) collide modulo T at T=121, G=12
    def bad_anchors(T, C, W, step):
        G = C - W
        Tper = -(-T // G)
        return sorted({(step + k * Tper) % T for k in range(G)})

    monkeypatch.setattr(OL, "anchors", bad_anchors)
    with pytest.raises(AssertionError):
        test_workload_anchor_figures(121, 21, 9, 12, 11, 11)


def test_mistake_left_first_extension_is_caught(monkeypatch):
    def left_first(t, T, C, W, step):
        if C >= T:
            return list(range(T))
        G = set(OL.anchors(T, C, W, step))
        lo, hi = OL.window(t, T, W)
        A = G | set(range(lo, hi + 1))
        right = False
        while len(A) < C:
            if right:
                while hi < T - 1:
                    hi += 1
                    if hi not in A:
                        A.add(hi)
                        break
            else:
                while lo > 0:
                    lo -= 1
                    if lo not in A:
                        A.add(lo)
                        break
            right = not right
        return sorted(A)

    monkeypatch.setattr(OL, "frame_set", left_first)
    with pytest.raises(AssertionError):
        test_worked_example_matches()


def test_mistake_rotation_mod_period_is_caught(monkeypatch):
    orig = OL.anchors

    def mod_period(T, C, W, step):
        return orig(T, C, W, step % OL.anchor_period(T, C, W))

    monkeypatch.setattr(OL, "anchors", mod_period)
    with pytest.raises(AssertionError):
        test_rotation_by_one_frame_per_step()


def test_mistake_window_not_shifted_is_caught(monkeypatch):
    def unshifted(t, T, W):
        lo = max(t - W // 2, 0)
        return lo, min(lo + W - 1, T - 1)

    monkeypatch.setattr(OL, "window", unshifted)
    with pytest.raises(AssertionError):
        test_invariants_brute_force()


def test_fixed_grid_ablation_never_covers_intermediate_frames():
    # the non-rotating pattern the pages contrast with (gist.science summary, "Rotating Global
    # Anchors": a fixed grid leaves intermediate frames seen only locally): holding the step at 0,
    # only the G grid frames are ever anchors; with rotation every frame is, within T_per steps
    T, C, W = 121, 21, 9
    G, Tper = C - W, OL.anchor_period(T, C, W)
    fixed = [0] * T
    for _ in range(Tper):
        for f in OL.anchors(T, C, W, 0):
            fixed[f] += 1
    assert sum(1 for c in fixed if c == 0) == T - G
    assert min(OL.anchor_coverage(T, C, W, 0)) >= 1
