"""Plain CPU oracle for LVSA frame-granular block-sparse attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library under ``block_sparse_attention_frame_b200/`` and
imports nothing from it.

Contents
--------
``lists``      frame sets A(t) = G_s U W(t) enumerated by definition (Python
               sets, pure integer work), plus the invariant checkers the pages
               state (budget, anchor count, rotation, coverage).
``attention``  softmax attention restricted to the frames of A(t), in float64
               with numpy, a separate plain dense attention routine, and the
               joint video + text form (text tokens after the video).

Sources (pages on "LVSA: Training-Free Sparse Attention for Long Video
Diffusion"):
  * gist.science technical summary, section 2 "Methodology", "Core Mechanism":
    A(t) = G U W(t); "Rotating Global Anchors": G_s shifts with the denoising
    step, every frame is an anchor within T_per steps; "Expanded Adaptive
    Windows": window of W frames extended so |A(t)| ~ C; "Complexity":
    O(T * C * P^2 * d).
  * techwalker article (Huawei Paris research, "不再原地打转"), section 二:
    T_per ~ T / (C - W); the window grows toward the sequence ends with new
    non-overlapping frames until the target count is reached.  Section 三:
    anchors move one frame per step modulo the total frame count; the anchor
    count is the same at every step; a few frames may be an anchor one extra
    time when T is not a multiple of the stride.

Readings where the pages are silent or disagree:
  * rotation offset is ``step mod T`` (section 三 of the techwalker article);
  * anchors sit at the fractional stride floor(k*T/G), k = 0..G-1, so there
    are always G distinct anchors;
  * the window for even W is [t - W//2, t - W//2 + W - 1], shifted inward at
    the ends;
  * extension alternates right/left, right first, one new non-anchor frame per
    turn, skipping a side that reached the sequence end;
  * C >= T means every query frame attends to all T frames (dense);
  * one joint softmax over all selected tokens, scale 1/sqrt(d) by default;
  * text tokens of a joint video + text sequence (pages silent; HunyuanVideo
    1.5 is named as dual-stream in the techwalker article, section 四): every
    video query attends them besides A(t), and a text query attends every
    token.

Parity status: every function here is pinned by tests in
``tests/test_oracle_lists.py``, ``tests/test_oracle_attention.py`` and
``tests/test_oracle_joint.py``
(hand-derived worked example, brute-force invariants, closed forms and a
library masked-attention routine).  No function is "parity unpinned".
"""

from . import lists, attention  # noqa: F401
