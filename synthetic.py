"""Seeded synthetic inputs shaped like the LVSA workloads.

This module holds no attention or frame-selection arithmetic: it only draws
random tensors.  It is the one piece shared by the CUDA path's callers and by
the oracle's callers (both receive the tensors it returns).

Workloads (latent frames T x tokens per frame P, heads H, head dim d, budget C,
window W).  P = 1560 = 30 x 52 patches of a 480x832 video; C follows the
pages' rule "budget = training horizon in latent frames" (81 frames / VAE
factor 4 -> 21; 129 frames -> 33).  The pages measure real model activations,
which are not available; these draws stand in for them:

* Q, V ~ N(0, 1)
* K = mu[b, frame, head, :] + N(0, 1) token noise, mu ~ 0.5 * N(0, 1)
  (a per-frame mean vector with standard deviation 0.5, so keys of one frame
  are correlated the way patch keys of one video frame are)
* drawn in the order mu, Q, K-noise, V from one ``torch.Generator`` seeded
  with ``seed``; the tiny case draws fp32 Q, K, V ~ N(0, 1) in that order on
  the CPU.

All tensors are laid out [batch, T*P, heads, d] (frame-major tokens).
"""

from __future__ import annotations

from dataclasses import dataclass, asdict

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    P: int
    H: int
    d: int
    C: int
    W: int
    B: int = 1
    seed: int = 0
    steps: int = 50
    frame_correlated_k: bool = True

    @property
    def L(self) -> int:
        return min(self.C, self.T)

    @property
    def tokens(self) -> int:
        return self.T * self.P

    def as_dict(self) -> dict:
        return asdict(self)


WORKLOADS = {
    # tiny correctness case: fp32 N(0,1) Q/K/V, rounded to bf16 for the kernel
    "tiny": Workload("tiny", T=8, P=64, H=2, d=64, C=4, W=2, seed=0, steps=8,
                     frame_correlated_k=False),
    # Wan-2.1-1.3B at its 1x training horizon: C = T, LVSA equals dense
    "wan1.3b_1x": Workload("wan1.3b_1x", T=21, P=1560, H=12, d=128, C=21, W=9, seed=1002, steps=1),
    # Wan-2.1-1.3B at 6x horizon (481 video frames = 121 latent frames)
    "wan1.3b_6x": Workload("wan1.3b_6x", T=121, P=1560, H=12, d=128, C=21, W=9, seed=1003),
    # Wan-2.1-14B at 6x horizon
    "wan14b_6x": Workload("wan14b_6x", T=121, P=1560, H=40, d=128, C=21, W=9, seed=1004),
    # HunyuanVideo-1.5 at 1.5x horizon (193 video frames = 49 latent frames)
    "hunyuan1.5_1.5x": Workload("hunyuan1.5_1.5x", T=49, P=1560, H=16, d=128, C=33, W=13, seed=1005),
    # HunyuanVideo-1.5 at 2x horizon (257 video frames = 65 latent frames; the pages' out-of-memory case for
    # dense attention in the full model on an 80 GB GPU)
    "hunyuan1.5_2x": Workload("hunyuan1.5_2x", T=65, P=1560, H=16, d=128, C=33, W=13, seed=1006),
    # profiling slice: the Wan-1.3B 6x call with 2 of its 12 heads (Q+K+V+O = 387 MB, still > L2)
    "wan1.3b_6x_h2": Workload("wan1.3b_6x_h2", T=121, P=1560, H=2, d=128, C=21, W=9, seed=1003),
}


def make_qkv(w: Workload, device="cpu", dtype=torch.bfloat16, seed: int | None = None):
    """Draw (q, k, v) for workload ``w`` on ``device``.

    For the tiny case the fp32 draws are returned rounded to ``dtype``; pass
    ``dtype=torch.float32`` to get the unrounded values.
    """
    seed = w.seed if seed is None else seed
    shape = (w.B, w.tokens, w.H, w.d)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    if not w.frame_correlated_k:
        q = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        k = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        v = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        return q.to(dtype), k.to(dtype), v.to(dtype)
    mu = 0.5 * torch.randn((w.B, w.T, 1, w.H, w.d), generator=g, device=device, dtype=torch.float32)
    q = torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(dtype)
    k = torch.randn((w.B, w.T, w.P, w.H, w.d), generator=g, device=device, dtype=torch.float32)
    k = (k + mu).reshape(shape).to(dtype)
    v = torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(dtype)
    return q, k, v


def make_custom(T: int, P: int, H: int, d: int, B: int = 1, seed: int = 0, device="cpu",
                dtype=torch.bfloat16, frame_correlated_k: bool = True):
    """Same recipe for an arbitrary shape (parity cases at other sizes)."""
    w = Workload("custom", T=T, P=P, H=H, d=d, C=T, W=1, B=B, seed=seed,
                 frame_correlated_k=frame_correlated_k)
    return make_qkv(w, device=device, dtype=dtype)


def make_joint(T: int, P: int, n_text: int, H: int, d: int, B: int = 1, seed: int = 0, device="cpu",
               dtype=torch.bfloat16):
    """A joint video + text sequence [batch, T*P + n_text, heads, d]: the video tokens drawn as
    ``make_custom``, then n_text text tokens with Q, K, V ~ N(0, 1) from a generator seeded with seed + 1,
    drawn in the order Q, K, V.  (HunyuanVideo 1.5 encodes its prompt into up to a few hundred text
    tokens; their statistics are not available either.)"""
    q, k, v = make_custom(T, P, H, d, B=B, seed=seed, device=device, dtype=dtype)
    g = torch.Generator(device=device)
    g.manual_seed(seed + 1)
    shape = (B, n_text, H, d)
    tq, tk, tv = (torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(dtype) for _ in range(3))
    return torch.cat([q, tq], dim=1), torch.cat([k, tk], dim=1), torch.cat([v, tv], dim=1)
