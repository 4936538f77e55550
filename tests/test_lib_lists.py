"""The library's host list builder (C ABI) against the oracle: bit-exact.

The library computes the lists in closed form (prefix counts of non-anchor
frames); the oracle enumerates sets turn by turn.  They share no code.
"""

import numpy as np
import pytest

from oracle import lists as OL

WORKLOAD_PARAMS = [  # (T, C, W) of the five workloads
    (8, 4, 2), (21, 21, 9), (121, 21, 9), (121, 21, 9), (49, 33, 13),
]


@pytest.mark.parametrize("T,C,W", sorted(set(WORKLOAD_PARAMS)))
def test_workload_lists_bit_exact_steps_0_to_49(lib, T, C, W):
    for s in range(50):
        got = lib.lvsa_build_frame_lists(T, C, W, s)
        assert got.dtype == np.int32 and got.shape == (T, min(C, T))
        assert got.tolist() == OL.frame_lists(T, C, W, s), (T, C, W, s)
        if C < T and C > W:
            assert lib.lvsa_build_anchors(T, C, W, s).tolist() == OL.anchors(T, C, W, s)


def test_small_sweep_bit_exact(lib):
    n = 0
    for T in range(1, 15):
        for C in range(1, T + 2):
            for W in range(1, C + 1):
                for s in range(0, T + 2):
                    assert lib.lvsa_build_frame_lists(T, C, W, s).tolist() == OL.frame_lists(T, C, W, s), \
                        (T, C, W, s)
                    n += 1
    assert n > 3000


@pytest.mark.parametrize("T,C,W", [(257, 21, 9), (65, 33, 13), (161, 21, 9), (200, 40, 1), (97, 96, 3)])
def test_longer_horizons_bit_exact(lib, T, C, W):
    for s in (0, 1, 7, T - 1, T, 3 * T + 5, 10**12 + 3):
        assert lib.lvsa_build_frame_lists(T, C, W, s).tolist() == OL.frame_lists(T, C, W, s)


def test_errors(lib):
    import ctypes

    for args in [(0, 4, 2, 0), (8, 0, 1, 0), (8, 4, 0, 0), (8, 4, 5, 0), (8, 4, 2, -1)]:
        with pytest.raises(lib.LvsaError) as e:
            lib.lvsa_build_frame_lists(*args)
        assert e.value.status == lib.LVSA_ERR_INVALID_ARG
    # capacity too small: error, and L is still reported
    L = ctypes.c_int(0)
    buf = (ctypes.c_int32 * 10)()
    st = lib._lib.lvsa_build_frame_lists(8, 4, 2, 0, buf, 10, ctypes.byref(L))
    assert st == lib.LVSA_ERR_BUFFER_TOO_SMALL and L.value == 4


def test_random_parameters_bit_exact(lib):
    """Seeded random (T, C, W, step), including far steps and budgets at or above T."""
    g = np.random.default_rng(2026)
    for _ in range(300):
        T = int(g.integers(1, 700))
        C = int(g.integers(1, T + 3))
        W = int(g.integers(1, C + 1))
        s = int(g.integers(0, 10**9))
        assert lib.lvsa_build_frame_lists(T, C, W, s).tolist() == OL.frame_lists(T, C, W, s), (T, C, W, s)


def test_pipeline_lists_rotating_and_fixed_grid(lib):
    """The per-step pipeline's host lists: step s's lists when the anchors rotate; the step-0 lists at every
    step in the fixed-grid ablation (anchors that never move)."""
    from block_sparse_attention_frame_b200 import pipeline

    T, C, W = 121, 21, 9
    step0 = OL.frame_lists(T, C, W, 0)
    for s in range(50):
        rot = pipeline.host_lists(T, C, W, s)
        fixed = pipeline.host_lists(T, C, W, s, fixed_grid=True)
        assert rot.tolist() == OL.frame_lists(T, C, W, s)
        assert fixed.tolist() == step0
        assert pipeline.list_step(s, True) == 0 and pipeline.list_step(s, False) == s
        if s % T != 0:
            assert rot.tolist() != step0
