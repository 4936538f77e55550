"""Pins for the oracle's torch-tensor inputs (no GPU, no library).

The GPU parity tests hand the oracle host torch tensors (bf16 as the kernel reads them, or fp32), while the
oracle's other pins feed numpy float64 arrays.  These tests pin the torch branch to the numpy one: the same
values, widened to float64 here by a route of their own (bf16 bit patterns shifted into float32), must give
results equal to the last bit, for every attention function of the oracle.  Planted mistakes in the torch
gather (wrong head, wrong batch entry, tokens one late) and in the widening (through float16) must fail.
A tensor in device memory must be refused.
"""

import numpy as np
import pytest
import torch

from oracle import attention as OA
from oracle import lists as OL

B, T, P, H, D = 2, 5, 4, 3, 8
N_TEXT = 3


def bf16_to_f64(x: torch.Tensor) -> np.ndarray:
    """bf16 -> float64 from the bit patterns: a bf16 value is the upper half of a float32."""
    bits = x.contiguous().view(torch.int16).numpy().astype(np.uint16).astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


def draws(tokens, seed, dtype, scale=1.5):
    g = torch.Generator().manual_seed(seed)
    xs = [(torch.randn((B, tokens, H, D), generator=g) * scale).to(dtype) for _ in range(3)]
    if dtype == torch.bfloat16:
        return xs, [bf16_to_f64(x) for x in xs]
    return xs, [x.numpy().astype(np.float64) for x in xs]


def assert_same(a, b):
    assert a.shape == b.shape
    assert np.array_equal(a, b), float(np.abs(a - b).max())


def call_all(xs, lists):
    q, k, v = xs
    rows = [1, 3, 4, 9, 10, 17, 19]  # frames 0, 0, 1, 2, 2, 4, 4
    return [
        OA.sparse_attention_rows(q, k, v, lists, P, rows),
        OA.sparse_attention(q, k, v, lists, P),
        OA.dense_attention(q[:, :T * P], k[:, :T * P], v[:, :T * P]),
    ]


def call_joint(xs, lists):
    q, k, v = xs
    rows = [0, 5, 11, 19, 20, 22]  # video rows of frames 0, 1, 2, 4 and two text rows
    return [OA.joint_attention_rows(q, k, v, lists, P, T, rows), OA.joint_attention(q, k, v, lists, P, T)]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_torch_inputs_equal_numpy_inputs(dtype):
    lists = OL.frame_lists(T, 3, 1, 2)
    xs, ns = draws(T * P, seed=7, dtype=dtype)
    for a, b in zip(call_all(xs, lists), call_all(ns, lists)):
        assert_same(a, b)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_joint_torch_inputs_equal_numpy_inputs(dtype):
    lists = OL.frame_lists(T, 3, 1, 4)
    xs, ns = draws(T * P + N_TEXT, seed=8, dtype=dtype)
    for a, b in zip(call_joint(xs, lists), call_joint(ns, lists)):
        assert_same(a, b)


def test_bit_widening_is_the_plain_conversion():
    # the test's own bf16 -> float64 route agrees with torch's on values across the bf16 range
    x = torch.tensor([0.0, -0.0, 1.0, -3.5, 1e-30, 3e38, 2 ** -130, 123.456]).to(torch.bfloat16)
    assert np.array_equal(bf16_to_f64(x), x.to(torch.float64).numpy())


def _planted_takes():
    def wrong_head(x, b, tokens, h):
        if hasattr(x, "detach"):
            idx = torch.as_tensor(tokens, dtype=torch.long)
            return x[b].index_select(0, idx)[:, (h + 1) % x.shape[2], :].to(torch.float64).numpy()
        return np.asarray(x[b, tokens, h, :], dtype=np.float64)

    def wrong_batch(x, b, tokens, h):
        if hasattr(x, "detach"):
            idx = torch.as_tensor(tokens, dtype=torch.long)
            return x[(b + 1) % x.shape[0]].index_select(0, idx)[:, h, :].to(torch.float64).numpy()
        return np.asarray(x[b, tokens, h, :], dtype=np.float64)

    def token_late(x, b, tokens, h):
        if hasattr(x, "detach"):
            idx = torch.as_tensor(np.minimum(np.asarray(tokens) + 1, x.shape[1] - 1), dtype=torch.long)
            return x[b].index_select(0, idx)[:, h, :].to(torch.float64).numpy()
        return np.asarray(x[b, tokens, h, :], dtype=np.float64)

    def via_half(x, b, tokens, h):
        if hasattr(x, "detach"):
            idx = torch.as_tensor(tokens, dtype=torch.long)
            return x[b].index_select(0, idx)[:, h, :].to(torch.float16).to(torch.float64).numpy()
        return np.asarray(x[b, tokens, h, :], dtype=np.float64)

    return [wrong_head, wrong_batch, token_late, via_half]


@pytest.mark.parametrize("plant", _planted_takes(), ids=lambda f: f.__name__)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_planted_gather_mistakes_fail(monkeypatch, plant, dtype):
    lists = OL.frame_lists(T, 3, 1, 2)
    # values below float16's normal range, so that the float16 plant loses bits of them for both input types
    xs, ns = draws(T * P, seed=9, dtype=dtype, scale=1e-6)
    ref = OA.sparse_attention_rows(ns[0], ns[1], ns[2], lists, P, range(T * P))
    assert_same(OA.sparse_attention_rows(xs[0], xs[1], xs[2], lists, P, range(T * P)), ref)
    monkeypatch.setattr(OA, "_take", plant)
    got = OA.sparse_attention_rows(xs[0], xs[1], xs[2], lists, P, range(T * P))
    assert not np.array_equal(got, ref)


def test_device_tensors_are_refused():
    x = torch.zeros((1, 4, 1, 8), device="meta")
    with pytest.raises(ValueError, match="host tensors only"):
        OA.sparse_attention_rows(x, x, x, [[0]], 4, [0])
    with pytest.raises(ValueError, match="host tensors only"):
        OA.dense_attention(x, x, x)
