"""Oracle: softmax attention restricted to the LVSA frame sets (test infrastructure).

gist.science technical summary, section 2 "Core Mechanism" and "Complexity":
a query token of frame t attends only to the tokens of the frames in A(t),
costing O(C * P * d) per query.  Reading (the pages are silent on it): one
softmax over all selected tokens together, scale 1/sqrt(d) by default.

For query token i of frame t, with J(t) the tokens of the frames in A(t):

    O_i = sum_{j in J(t)} exp(sigma * q_i . k_j - m_i) v_j
          / sum_{j in J(t)} exp(sigma * q_i . k_j - m_i)

with m_i the row maximum (subtracted for range only; it cancels exactly).

Layout of every tensor: [batch, T * P, heads, d], frame-major tokens (token
t*P + i is patch i of latent frame t).  All arithmetic is float64 numpy; a
matrix product is the only library primitive used.
"""

from __future__ import annotations

import math

import numpy as np


def _host_tensor(x):
    """A torch tensor given to the oracle must already be in host memory: the oracle never touches a GPU."""
    if x.device.type != "cpu":
        raise ValueError(f"the oracle takes host tensors only (got one on {x.device}); pass x.cpu()")
    return x


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor (host memory, any float dtype) -> float64 numpy
        import torch

        x = _host_tensor(x).detach().to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _take(x, b: int, tokens: np.ndarray, h: int) -> np.ndarray:
    """x[b, tokens, h, :] as float64.  A torch tensor (host memory) is gathered
    before it is widened, so a large bf16 tensor is never converted whole; the
    widening bf16/fp32 -> float64 is exact either way."""
    if hasattr(x, "detach"):
        import torch

        idx = torch.as_tensor(tokens, dtype=torch.long)
        return _host_tensor(x)[b].index_select(0, idx)[:, h, :].detach().to(torch.float64).numpy()
    return np.asarray(x[b, tokens, h, :], dtype=np.float64)


def default_scale(d: int) -> float:
    """1/sqrt(d), the usual DiT self-attention scale (pages silent)."""
    return 1.0 / math.sqrt(d)


def frame_tokens(frames, P: int) -> np.ndarray:
    """Token indices of the given frames, each frame counted once, ascending."""
    fs = sorted(set(int(f) for f in frames))
    return np.concatenate([np.arange(f * P, (f + 1) * P) for f in fs]) if fs else np.zeros(0, np.int64)


def sparse_attention_rows(q, k, v, lists, P: int, rows, scale: float | None = None) -> np.ndarray:
    """O for the query tokens ``rows`` (iterable of token indices) of every
    batch and head.

    ``q, k, v``: numpy arrays or torch tensors [batch, T*P, heads, d].
    ``lists[t]`` is the frame set A(t) of query frame t.  Returns float64
    [batch, len(rows), heads, d].
    """
    B, Ltok, H, d = q.shape
    sigma = default_scale(d) if scale is None or scale <= 0 else float(scale)
    rows = np.asarray(list(rows), dtype=np.int64)
    out = np.zeros((B, rows.size, H, d), dtype=np.float64)
    frames_of_rows = rows // P
    for t in np.unique(frames_of_rows):
        sel = np.nonzero(frames_of_rows == t)[0]
        toks = frame_tokens(lists[int(t)], P)
        for b in range(B):
            for h in range(H):
                Q = _take(q, b, rows[sel], h)      # [r, d]
                K = _take(k, b, toks, h)           # [n, d]
                V = _take(v, b, toks, h)           # [n, d]
                S = sigma * (Q @ K.T)              # [r, n]
                m = S.max(axis=1, keepdims=True)
                E = np.exp(S - m)
                out[b, sel, h, :] = (E @ V) / E.sum(axis=1, keepdims=True)
    return out


def sparse_attention(q, k, v, lists, P: int, scale: float | None = None) -> np.ndarray:
    """O for every query token: float64 [batch, T*P, heads, d]."""
    Ltok = q.shape[1]
    return sparse_attention_rows(q, k, v, lists, P, range(Ltok), scale)


def dense_attention(q, k, v, scale: float | None = None) -> np.ndarray:
    """Plain full softmax attention over all tokens (the dense baseline the
    pages compare against), float64 [batch, tokens, heads, d]."""
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, Ltok, H, d = q.shape
    sigma = default_scale(d) if scale is None or scale <= 0 else float(scale)
    out = np.zeros_like(q)
    for b in range(B):
        for h in range(H):
            S = sigma * (q[b, :, h, :] @ k[b, :, h, :].T)
            S = S - S.max(axis=1, keepdims=True)
            E = np.exp(S)
            out[b, :, h, :] = (E @ v[b, :, h, :]) / E.sum(axis=1, keepdims=True)
    return out



def joint_token_set(t: int, lists, P: int, T: int, n_text: int) -> np.ndarray:
    """Keys of a query token of latent frame t in a joint video + text sequence (tokens [0, T*P) are the
    video, frame-major; [T*P, T*P + n_text) the text).  The pages only define the video part, A(t)
    (gist.science summary, section 2 "Core Mechanism"); reading for the text (pages silent): every video
    query also attends every text token.  A text query (t >= T) attends every token."""
    text = np.arange(T * P, T * P + n_text, dtype=np.int64)
    if t >= T:
        return np.arange(0, T * P + n_text, dtype=np.int64)
    return np.concatenate([frame_tokens(lists[int(t)], P), text])


def joint_attention_rows(q, k, v, lists, P: int, T: int, rows, scale: float | None = None) -> np.ndarray:
    """O for the query tokens ``rows`` of a joint sequence [batch, T*P + n_text, heads, d] (n_text taken
    from the tensors): one softmax over joint_token_set of each row.  float64 [batch, len(rows), heads, d]."""
    B, Ltok, H, d = q.shape
    n_text = Ltok - T * P
    if n_text < 0:
        raise ValueError("tensors hold fewer than T*P tokens")
    sigma = default_scale(d) if scale is None or scale <= 0 else float(scale)
    rows = np.asarray(list(rows), dtype=np.int64)
    out = np.zeros((B, rows.size, H, d), dtype=np.float64)
    group = np.minimum(rows // P, T)  # the frame of a video row; T for every text row
    for t in np.unique(group):
        sel = np.nonzero(group == t)[0]
        toks = joint_token_set(int(t), lists, P, T, n_text)
        for b in range(B):
            for h in range(H):
                Q = _take(q, b, rows[sel], h)
                K = _take(k, b, toks, h)
                V = _take(v, b, toks, h)
                S = sigma * (Q @ K.T)
                m = S.max(axis=1, keepdims=True)
                E = np.exp(S - m)
                out[b, sel, h, :] = (E @ V) / E.sum(axis=1, keepdims=True)
    return out


def joint_attention(q, k, v, lists, P: int, T: int, scale: float | None = None) -> np.ndarray:
    """O for every token of a joint video + text sequence: float64 [batch, T*P + n_text, heads, d]."""
    return joint_attention_rows(q, k, v, lists, P, T, range(q.shape[1]), scale)
