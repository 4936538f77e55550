"""Pins for the oracle's attention (no GPU, no library).

What pins what:
* a library routine: torch's scaled_dot_product_attention in float64 on the CPU,
  given the dense token mask expanded from the frame lists, must equal the
  oracle (sparse case) and, unmasked, the oracle's dense routine (C >= T);
* closed forms: equal keys -> the plain mean of V over the selected tokens; with
  V carrying a one-hot marker of each token's frame that mean shows exactly which
  frames are attended, each once; one dominant key -> its value row; adding a
  constant vector to every key changes nothing; list order does not matter;
* T = 1 is ordinary attention over one frame;
* planted mistakes (wrong scale, a frame counted twice, transposed product, per-frame
  softmax, frame tokens off by one, the previous frame's list)
  must fail one of the above.
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import attention as OA
from oracle import lists as OL


def rand_qkv(B, T, P, H, d, seed):
    g = np.random.default_rng(seed)
    shape = (B, T * P, H, d)
    return g.standard_normal(shape), g.standard_normal(shape), g.standard_normal(shape)


def sdpa_masked(q, k, v, lists, P, scale=None):
    """Library masked attention: token mask = frame mask expanded P x P."""
    B, Ltok, H, d = q.shape
    T = Ltok // P
    fmask = np.zeros((T, T), dtype=bool)
    for t, row in enumerate(lists):
        fmask[t, list(row)] = True
    tmask = np.kron(fmask, np.ones((P, P), dtype=bool))
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k).permute(0, 2, 1, 3)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3)
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(tmask), scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


def sdpa_dense(q, k, v, scale=None):
    qt, kt, vt = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    return F.scaled_dot_product_attention(qt, kt, vt, scale=scale).permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("T,P,H,d,C,W,step", [
    (8, 5, 2, 8, 4, 2, 0), (8, 5, 2, 8, 4, 2, 3), (9, 4, 1, 16, 5, 2, 7),
    (12, 3, 2, 8, 6, 3, 11), (7, 6, 1, 4, 3, 3, 2), (10, 2, 3, 8, 4, 1, 5),
])
def test_sparse_matches_library_masked_attention(T, P, H, d, C, W, step):
    q, k, v = rand_qkv(2, T, P, H, d, seed=T * 100 + step)
    lists = OL.frame_lists(T, C, W, step)
    ref = sdpa_masked(q, k, v, lists, P)
    got = OA.sparse_attention(q, k, v, lists, P)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


def test_explicit_scale_matches_library():
    q, k, v = rand_qkv(1, 6, 4, 2, 8, seed=5)
    lists = OL.frame_lists(6, 3, 1, 4)
    np.testing.assert_allclose(OA.sparse_attention(q, k, v, lists, 4, scale=0.77),
                               sdpa_masked(q, k, v, lists, 4, scale=0.77), rtol=1e-11, atol=1e-12)


def test_dense_budget_equals_dense_attention():
    T, P = 6, 5
    q, k, v = rand_qkv(1, T, P, 2, 8, seed=11)
    lists = OL.frame_lists(T, T, 3, 9)
    dense = OA.dense_attention(q, k, v)
    np.testing.assert_allclose(OA.sparse_attention(q, k, v, lists, P), dense, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dense, sdpa_dense(q, k, v), rtol=1e-11, atol=1e-12)


def test_single_frame_is_plain_attention():
    q, k, v = rand_qkv(1, 1, 37, 2, 16, seed=3)
    lists = OL.frame_lists(1, 21, 9, 0)
    assert lists == [[0]]
    np.testing.assert_allclose(OA.sparse_attention(q, k, v, lists, 37), sdpa_dense(q, k, v),
                               rtol=1e-11, atol=1e-12)


def marker_inputs(T, P, d):
    """Equal (zero) keys and V rows that are one-hot in the token's frame."""
    assert d >= T
    q = np.random.default_rng(0).standard_normal((1, T * P, 1, d))
    k = np.zeros((1, T * P, 1, d))
    v = np.zeros((1, T * P, 1, d))
    for tok in range(T * P):
        v[0, tok, 0, tok // P] = 1.0
    return q, k, v


@pytest.mark.parametrize("T,C,W,step", [(8, 4, 2, 0), (8, 4, 2, 1), (11, 5, 2, 6), (9, 9, 3, 0), (10, 4, 4, 2)])
def test_equal_keys_give_uniform_weights_over_selected_frames(T, C, W, step):
    P, d = 3, 16
    q, k, v = marker_inputs(T, P, d)
    lists = OL.frame_lists(T, C, W, step)
    out = OA.sparse_attention(q, k, v, lists, P)
    for t in range(T):
        expect = np.zeros(d)
        expect[lists[t]] = 1.0 / len(lists[t])
        for i in range(P):
            np.testing.assert_allclose(out[0, t * P + i, 0], expect, atol=1e-14)


def test_dominant_key_selects_its_value():
    # every frame f holds one large key whose logit grows with f; a query of
    # frame t must pick the value of the largest frame IN A(t), ignoring the
    # even larger keys of frames outside A(t)
    T, P, d = 9, 4, 8
    q, k, v = rand_qkv(1, T, P, 1, d, seed=2)
    lists = OL.frame_lists(T, 4, 2, 1)
    q[0, :, 0, :] = 1.0
    for f in range(T):
        k[0, f * P + 2, 0, :] = 10.0 * (f + 1)
    out = OA.sparse_attention(q, k, v, lists, P)
    for t in range(T):
        expect = v[0, max(lists[t]) * P + 2, 0, :]
        np.testing.assert_allclose(out[0, t * P:(t + 1) * P, 0, :], np.broadcast_to(expect, (P, d)), atol=1e-9)
    assert any(max(lists[t]) < T - 1 for t in range(T))


def test_key_shift_invariance_and_list_order():
    T, P = 7, 4
    q, k, v = rand_qkv(1, T, P, 2, 8, seed=9)
    lists = OL.frame_lists(T, 4, 2, 3)
    base = OA.sparse_attention(q, k, v, lists, P)
    # q.(k + c) = q.k + q.c is a per-row constant: softmax ignores it
    c = np.random.default_rng(1).standard_normal(8)
    np.testing.assert_allclose(OA.sparse_attention(q, k + c, v, lists, P), base, rtol=1e-10, atol=1e-12)
    rev = [list(reversed(r)) for r in lists]
    np.testing.assert_allclose(OA.sparse_attention(q, k, v, rev, P), base, rtol=1e-12, atol=1e-14)


def test_rows_subset_equals_full():
    T, P = 6, 5
    q, k, v = rand_qkv(2, T, P, 2, 8, seed=4)
    lists = OL.frame_lists(T, 3, 2, 2)
    full = OA.sparse_attention(q, k, v, lists, P)
    rows = [0, 4, 5, 13, 29]
    np.testing.assert_allclose(OA.sparse_attention_rows(q, k, v, lists, P, rows), full[:, rows], rtol=1e-13)


# ----------------------------------------------------------------------------
# Planted mistakes (monkeypatched into the oracle, CPU only)
# ----------------------------------------------------------------------------

def test_mistake_wrong_scale_is_caught(monkeypatch):
    monkeypatch.setattr(OA, "default_scale", lambda d: 1.0 / d)
    with pytest.raises(AssertionError):
        test_sparse_matches_library_masked_attention(8, 5, 2, 8, 4, 2, 0)


def test_mistake_double_counted_frame_is_caught(monkeypatch):
    def dup_tokens(frames, P):
        fs = [int(f) for f in frames]
        fs = fs + fs[:1]  # first frame counted twice
        return np.concatenate([np.arange(f * P, (f + 1) * P) for f in fs])

    monkeypatch.setattr(OA, "frame_tokens", dup_tokens)
    with pytest.raises(AssertionError):
        test_equal_keys_give_uniform_weights_over_selected_frames(8, 4, 2, 0)


def test_mistake_transposed_product_is_caught(monkeypatch):
    orig = OA.sparse_attention_rows

    def transposed(q, k, v, lists, P, rows, scale=None):
        return orig(k, q, v, lists, P, rows, scale)  # q and k swapped

    monkeypatch.setattr(OA, "sparse_attention_rows", transposed)
    with pytest.raises(AssertionError):
        test_sparse_matches_library_masked_attention(8, 5, 2, 8, 4, 2, 0)


def test_mistake_per_frame_softmax_is_caught(monkeypatch):
    """A softmax normalised within each frame (and the frames then averaged) instead of one joint softmax."""

    def per_frame(q, k, v, lists, P, rows, scale=None):
        B, _, H, d = np.shape(q)
        q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
        sigma = OA.default_scale(d) if scale is None or scale <= 0 else scale
        rows = np.asarray(list(rows))
        out = np.zeros((B, rows.size, H, d))
        for n, r in enumerate(rows):
            frames = sorted(set(int(f) for f in lists[int(r) // P]))
            for b in range(B):
                for h in range(H):
                    acc = np.zeros(d)
                    for f in frames:
                        toks = np.arange(f * P, (f + 1) * P)
                        s = sigma * k[b, toks, h] @ q[b, r, h]
                        e = np.exp(s - s.max())
                        acc += (e / e.sum()) @ v[b, toks, h]
                    out[b, n, h] = acc / len(frames)
        return out

    monkeypatch.setattr(OA, "sparse_attention_rows", per_frame)
    with pytest.raises(AssertionError):
        test_sparse_matches_library_masked_attention(8, 5, 2, 8, 4, 2, 0)


def test_mistake_shifted_frame_tokens_is_caught(monkeypatch):
    """Frame f's tokens taken one token late (an off-by-one in the gather)."""

    def shifted(frames, P):
        fs = sorted(set(int(f) for f in frames))
        return np.concatenate([np.arange(f * P + 1, (f + 1) * P + 1) for f in fs]) % (8 * P)

    monkeypatch.setattr(OA, "frame_tokens", shifted)
    with pytest.raises(AssertionError):
        test_sparse_matches_library_masked_attention(8, 5, 2, 8, 4, 2, 0)


def test_mistake_previous_frame_list_is_caught(monkeypatch):
    """Query rows of frame t given the list of frame t - 1."""
    orig = OA.sparse_attention_rows

    def prev_list(q, k, v, lists, P, rows, scale=None):
        shifted = [lists[max(t - 1, 0)] for t in range(len(lists))]
        return orig(q, k, v, shifted, P, rows, scale)

    monkeypatch.setattr(OA, "sparse_attention_rows", prev_list)
    with pytest.raises(AssertionError):
        test_sparse_matches_library_masked_attention(8, 5, 2, 8, 4, 2, 0)
