"""Oracle: LVSA frame sets A(t) enumerated by definition (test infrastructure).

Each query frame t of a video with T latent frames attends to the frame set

    A(t) = G_s  U  E_s(t)

(gist.science technical summary, section 2 "Core Mechanism": A(t) = G U W(t)),
where G_s are the rotating global anchors of denoising step s and E_s(t) is the
local window W(t) after extension.  This module builds those sets the slow,
obvious way: Python sets, one frame at a time, in the order the pages describe
the steps.  It never reorders or batches the work.
"""

from __future__ import annotations


def check_args(T: int, C: int, W: int, step: int) -> None:
    """Parameter edges (pages are silent; reading: C, W, T >= 1, W <= C)."""
    if T < 1 or C < 1 or W < 1 or W > C or step < 0:
        raise ValueError(f"invalid LVSA parameters T={T} C={C} W={W} step={step}")


def anchor_count(T: int, C: int, W: int) -> int:
    """G = C - W anchors: the budget left after the window.

    techwalker article, section 二: the anchor spacing T_per is about T divided
    by the budget that remains after the window frames, C - W.
    """
    return C - W


def anchor_period(T: int, C: int, W: int) -> int:
    """T_per = ceil(T / G): the number of steps over which every frame is an
    anchor at least once (gist.science summary, "Rotating Global Anchors")."""
    G = anchor_count(T, C, W)
    if G <= 0:
        raise ValueError("no anchors (G = 0): anchor period undefined")
    return -(-T // G)


def anchors(T: int, C: int, W: int, step: int) -> list[int]:
    """Global anchor frames G_s of denoising step ``step``.

    Reading: G anchors at the fractional stride floor(k*T/G), k = 0..G-1, all
    shifted by ``step`` modulo T (techwalker article, section 三: the anchors
    move one frame per denoising step, wrapping modulo the total frame count).
    When G divides T this is the integer grid of stride T/G.
    """
    check_args(T, C, W, step)
    G = anchor_count(T, C, W)
    return sorted({(step + (k * T) // G) % T for k in range(G)})


def window(t: int, T: int, W: int) -> tuple[int, int]:
    """Local window of W frames centred on t, shifted inward at the ends.

    gist.science summary, "Expanded Adaptive Windows": each frame attends to a
    local temporal window of size W.  Reading for even W: lo = t - W//2.
    Returns the inclusive interval (lo, hi).
    """
    lo = t - W // 2
    hi = lo + W - 1
    if lo < 0:
        hi -= lo
        lo = 0
    if hi > T - 1:
        lo -= hi - (T - 1)
        hi = T - 1
    lo = max(lo, 0)
    return lo, hi


def frame_set(t: int, T: int, C: int, W: int, step: int) -> list[int]:
    """A(t) for query frame t at step ``step``, sorted ascending.

    1. C >= T: every frame (the budget covers the whole video, dense case).
    2. Otherwise A = G_s U [lo, hi] with the window from :func:`window`.
    3. Extension (techwalker article, section 二; gist.science summary,
       "Expanded Adaptive Windows"): while |A| < C, grow the window toward the
       sequence ends.  Turns alternate right, left, right, ...; on a turn the
       edge moves outward one frame at a time, passing anchor frames (already
       in A), until one new frame has been added or the sequence end is
       reached.  A side already at the sequence end is skipped.
    """
    check_args(T, C, W, step)
    if C >= T:
        return list(range(T))
    G = set(anchors(T, C, W, step))
    lo, hi = window(t, T, W)
    A = set(G) | set(range(lo, hi + 1))
    side_right = True
    while len(A) < C:
        if side_right:
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
        side_right = not side_right
    return sorted(A)


def frame_lists(T: int, C: int, W: int, step: int) -> list[list[int]]:
    """Per-query-frame KV frame lists: T rows of min(C, T) ascending frames."""
    check_args(T, C, W, step)
    return [frame_set(t, T, C, W, step) for t in range(T)]


# ---------------------------------------------------------------------------
# Invariant checkers (the properties the pages state), used by the tests.
# ---------------------------------------------------------------------------

def anchor_coverage(T: int, C: int, W: int, first_step: int) -> list[int]:
    """How often each frame is an anchor over T_per consecutive steps.

    gist.science summary, "Rotating Global Anchors": over T_per consecutive
    steps every frame serves as a global anchor; techwalker article, section
    三: a very few frames once more when T is not a multiple of the stride.
    """
    Tper = anchor_period(T, C, W)
    counts = [0] * T
    for s in range(first_step, first_step + Tper):
        for f in anchors(T, C, W, s):
            counts[f] += 1
    return counts
