"""The per-denoising-step path: host frame lists -> pinned buffer -> device -> sparse attention.

The method recomputes its sparsity pattern on the CPU at every denoising step: the anchors move one frame
per step (techwalker article "华为巴黎研究院让AI视频“不再原地打转”", sections 二 and 三; gist.science
summary, "Rotating Global Anchors").  ``StepPipeline.step(s, ...)`` runs one step of that loop:

1. ``lvsa_build_frame_lists(T, C, W, s)`` writes A(t) for every query frame straight into a page-locked
   host buffer (C ABI, a few microseconds at T = 121);
2. the buffer is copied to a device list buffer asynchronously on the caller's stream;
3. ``lvsa_attention`` runs on that stream.

Nothing here waits for the GPU in steady state, so the host work of step s+1 overlaps the kernel of step s.
Host and device list buffers form a ring of ``depth`` slots.  Before the host rewrites a slot it waits for
the event recorded after that slot's last copy.  A slot's device buffer is rewritten only by a copy queued
after every kernel that read it: the copies and the kernels of one stream run in order, and across
streams the copy waits for the event recorded after the kernel.

``fixed_grid=True`` is the ablation the pages contrast with rotation: the anchors never move, so every
step uses the step-0 pattern (gist.science summary, "Rotating Global Anchors").

NVTX ranges ``lvsa.build_lists``, ``lvsa.upload`` and ``lvsa.attention`` mark the three parts of a step
on a profiler timeline; with no profiler attached they cost a call each.
"""

from __future__ import annotations

import time

from . import lvsa_attention, lvsa_build_frame_lists


def list_step(step: int, fixed_grid: bool) -> int:
    """The step whose anchors a denoising step uses: itself, or 0 when the anchors do not rotate."""
    return 0 if fixed_grid else int(step)


def host_lists(T: int, C: int, W: int, step: int, fixed_grid: bool = False, out=None):
    """Frame lists of denoising step ``step`` as int32 [T, min(C, T)] (host), fixed-grid aware."""
    return lvsa_build_frame_lists(T, C, W, list_step(step, fixed_grid), out=out)


class StepPipeline:
    """One LVSA attention call per denoising step, the lists rebuilt on the host every step.

    T, C, W: latent frames, frame budget, window.  tokens_per_frame: P.  device: the CUDA device of the
    activations.  depth: slots of the host/device list ring (2 lets step s+1's build overlap step s).
    """

    def __init__(self, T: int, C: int, W: int, tokens_per_frame: int, device, fixed_grid: bool = False,
                 depth: int = 2):
        import torch

        if depth < 1:
            raise ValueError("depth >= 1")
        self.T, self.C, self.W, self.P = T, C, W, tokens_per_frame
        self.L = min(C, T)
        self.fixed_grid = fixed_grid
        self.device = torch.device(device)
        self.depth = depth
        self.host = [torch.empty((T, self.L), dtype=torch.int32).pin_memory() for _ in range(depth)]
        self.dev = [torch.empty((T, self.L), dtype=torch.int32, device=self.device) for _ in range(depth)]
        self.copied = [None] * depth  # event after the slot's last host -> device copy
        self.used = [None] * depth    # event after the last kernel that read the slot's device buffer
        self.build_us = []            # host list-build time of every step, microseconds
        self.calls = 0

    def step(self, step: int, q, k, v, out, stream=None, scale: float = 0.0, kernel_events=None):
        """Runs denoising step ``step``: lists of that step, upload, attention into ``out``.

        q, k, v, out: CUDA bf16 [batch, T*P, heads, d].  stream: a torch CUDA stream (default: the current
        one).  kernel_events: optional (start, end) torch CUDA events recorded around the kernel launch.
        Returns ``out``; asynchronous like ``lvsa_attention``.
        """
        import torch

        stream = torch.cuda.current_stream(self.device) if stream is None else stream
        i = self.calls % self.depth
        self.calls += 1
        if self.copied[i] is not None:
            self.copied[i].synchronize()  # the pinned buffer's previous copy has been read
        torch.cuda.nvtx.range_push("lvsa.build_lists")
        t0 = time.perf_counter()
        host_lists(self.T, self.C, self.W, step, self.fixed_grid, out=self.host[i].numpy())
        self.build_us.append((time.perf_counter() - t0) * 1e6)
        torch.cuda.nvtx.range_pop()
        torch.cuda.nvtx.range_push("lvsa.upload")
        with torch.cuda.stream(stream):
            if self.used[i] is not None:
                stream.wait_event(self.used[i])  # no kernel still reads the device buffer
            self.dev[i].copy_(self.host[i], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(stream)
            self.copied[i] = ev
        torch.cuda.nvtx.range_pop()
        torch.cuda.nvtx.range_push("lvsa.attention")
        if kernel_events is not None:
            kernel_events[0].record(stream)
        lvsa_attention(q, k, v, self.dev[i], self.P, scale=scale, out=out, stream=stream)
        if kernel_events is not None:
            kernel_events[1].record(stream)
        done = torch.cuda.Event()
        done.record(stream)
        self.used[i] = done
        torch.cuda.nvtx.range_pop()
        return out
