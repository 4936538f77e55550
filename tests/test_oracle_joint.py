"""Pins for the oracle's joint video + text attention (no GPU, no library).

Reading (the pages define A(t) for video frames only and are silent on other tokens): in a joint sequence
[video tokens of T frames, frame-major; n_text text tokens], a video query of frame t attends the tokens of
the frames in A(t) plus every text token, and a text query attends every token; one softmax per row.

What pins it:
* a library routine: torch's scaled_dot_product_attention in float64 with the token mask of that reading,
  built independently here from the frame lists;
* closed forms: with equal keys, V rows one-hot in the token's frame (and a separate channel for text
  tokens) give the plain mean over exactly the attended tokens;
* special cases: no text tokens is the video-only oracle; lists holding every frame is dense attention over
  the whole joint sequence;
* planted mistakes (text dropped from video rows, text rows limited to a frame list, text placed before
  the video) must fail one of the above.
"""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import attention as OA
from oracle import lists as OL


def rand_joint(B, T, P, n_text, H, d, seed):
    g = np.random.default_rng(seed)
    shape = (B, T * P + n_text, H, d)
    return g.standard_normal(shape), g.standard_normal(shape), g.standard_normal(shape)


def joint_mask(lists, T, P, n_text):
    L = T * P + n_text
    m = np.zeros((L, L), dtype=bool)
    for t in range(T):
        for f in set(int(x) for x in lists[t]):
            m[t * P:(t + 1) * P, f * P:(f + 1) * P] = True
        m[t * P:(t + 1) * P, T * P:] = True
    m[T * P:, :] = True
    return m


def sdpa(q, k, v, mask=None, scale=None):
    qt, kt, vt = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    am = None if mask is None else torch.from_numpy(mask)
    return F.scaled_dot_product_attention(qt, kt, vt, attn_mask=am, scale=scale).permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("T,P,n_text,H,d,C,W,step", [
    (8, 5, 3, 2, 8, 4, 2, 0), (8, 5, 7, 1, 8, 4, 2, 3), (9, 4, 1, 2, 16, 5, 2, 7), (6, 3, 10, 1, 8, 3, 1, 2),
])
def test_joint_matches_library_masked_attention(T, P, n_text, H, d, C, W, step):
    q, k, v = rand_joint(2, T, P, n_text, H, d, seed=T * 10 + n_text)
    lists = OL.frame_lists(T, C, W, step)
    got = OA.joint_attention(q, k, v, lists, P, T)
    np.testing.assert_allclose(got, sdpa(q, k, v, joint_mask(lists, T, P, n_text)), rtol=1e-11, atol=1e-12)
    got_s = OA.joint_attention(q, k, v, lists, P, T, scale=0.3)
    np.testing.assert_allclose(got_s, sdpa(q, k, v, joint_mask(lists, T, P, n_text), scale=0.3), rtol=1e-11,
                               atol=1e-12)


def test_no_text_is_the_video_oracle():
    T, P = 8, 4
    q, k, v = rand_joint(1, T, P, 0, 2, 8, seed=3)
    lists = OL.frame_lists(T, 4, 2, 5)
    np.testing.assert_allclose(OA.joint_attention(q, k, v, lists, P, T), OA.sparse_attention(q, k, v, lists, P),
                               rtol=0, atol=0)


def test_dense_lists_are_dense_joint_attention():
    T, P, n_text = 5, 3, 4
    q, k, v = rand_joint(1, T, P, n_text, 2, 8, seed=4)
    lists = OL.frame_lists(T, T, 1, 0)
    np.testing.assert_allclose(OA.joint_attention(q, k, v, lists, P, T), OA.dense_attention(q, k, v),
                               rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("T,C,W,step,n_text", [(8, 4, 2, 1, 5), (11, 5, 2, 6, 1), (7, 3, 3, 2, 9)])
def test_equal_keys_average_exactly_the_attended_tokens(T, C, W, step, n_text):
    P, d = 3, 16
    assert d >= T + 1
    L = T * P + n_text
    q = np.random.default_rng(1).standard_normal((1, L, 1, d))
    k = np.zeros((1, L, 1, d))
    v = np.zeros((1, L, 1, d))
    for tok in range(T * P):
        v[0, tok, 0, tok // P] = 1.0
    v[0, T * P:, 0, T] = 1.0  # text marker channel
    lists = OL.frame_lists(T, C, W, step)
    out = OA.joint_attention(q, k, v, lists, P, T)
    for t in range(T):
        n = len(set(lists[t])) * P + n_text
        expect = np.zeros(d)
        expect[sorted(set(lists[t]))] = P / n
        expect[T] = n_text / n
        for i in range(P):
            np.testing.assert_allclose(out[0, t * P + i, 0], expect, atol=1e-14)
    expect = np.zeros(d)
    expect[:T] = P / L
    expect[T] = n_text / L
    for i in range(n_text):
        np.testing.assert_allclose(out[0, T * P + i, 0], expect, atol=1e-14)


def _pins_hold(T=8, P=5, n_text=6, C=4, W=2, step=1):
    q, k, v = rand_joint(1, T, P, n_text, 2, 8, seed=9)
    lists = OL.frame_lists(T, C, W, step)
    return np.allclose(OA.joint_attention(q, k, v, lists, P, T), sdpa(q, k, v, joint_mask(lists, T, P, n_text)),
                       rtol=1e-10, atol=1e-11)


def test_mistake_text_dropped_from_video_rows_is_caught(monkeypatch):
    orig = OA.joint_token_set

    def no_text(t, lists, P, T, n_text):
        return orig(t, lists, P, T, 0) if t < T else orig(t, lists, P, T, n_text)

    monkeypatch.setattr(OA, "joint_token_set", no_text)
    assert not _pins_hold()


def test_mistake_text_rows_limited_to_a_frame_list_is_caught(monkeypatch):
    orig = OA.joint_token_set

    def text_as_last_frame(t, lists, P, T, n_text):
        return orig(min(t, T - 1), lists, P, T, n_text)

    monkeypatch.setattr(OA, "joint_token_set", text_as_last_frame)
    assert not _pins_hold()


def test_mistake_text_before_video_is_caught(monkeypatch):
    def text_first(t, lists, P, T, n_text):
        # text taken as the first n_text tokens, the video after it
        if t >= T:
            return np.arange(0, T * P + n_text, dtype=np.int64)
        return np.concatenate([np.arange(n_text), n_text + OA.frame_tokens(lists[int(t)], P)])

    monkeypatch.setattr(OA, "joint_token_set", text_first)
    assert not _pins_hold()
