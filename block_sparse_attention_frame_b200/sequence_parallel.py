"""Sequence-parallel LVSA attention over the GPUs of one node (DeepSpeed-Ulysses layout).

The method's multi-device setting (techwalker article "华为巴黎研究院让AI视频“不再原地打转”", section 五:
Wan 2.2-A14B on 8 NPUs with DeepSpeed-Ulysses sequence parallelism): every rank holds a token range of Q, K,
V and of the output, for every head.  Attention needs all tokens of a head, and heads are independent (A(t)
is indexed by query frame and step only and shared by every head: gist.science summary, section 2 "Core
Mechanism"), so each rank computes a band of heads over the whole sequence.  Both exchanges run in this
library's kernels over peer memory, with no collective library on the data path:

  sequence -> heads  ``lvsa_seq_to_heads`` reads the rank's band from every rank's range buffer through CUDA
                     IPC mappings (NVLink peer loads) into local band buffers;
  heads -> sequence  ``lvsa_attention_to_chunks`` stores every output row straight into the range buffer of
                     the rank that owns its token (peer stores from the attention epilogue).

The process group only orders the ranks: a barrier once the inputs are written and one after the attention;
no kernel waits on another GPU.  With one rank nothing is exchanged and the call is ``lvsa_attention``.

Layout: rank r's buffers ``q``, ``k``, ``v``, ``out`` are bf16 [batch, chunk_tokens[r], heads, d] and hold
tokens [start_r, start_r + chunk_tokens[r]) of the frame-major sequence (start_r = sum of the counts of the
ranks before r).  The caller writes its inputs into ``q``, ``k``, ``v`` and reads ``out`` after the call.
"""

from __future__ import annotations

from . import (lvsa_attention_host, lvsa_attention_to_chunks, lvsa_ipc_export, lvsa_ipc_import, lvsa_ipc_release,
               lvsa_seq_to_heads)


def head_band(rank: int, world: int, heads: int) -> tuple[int, int]:
    """Heads [h0, h0 + n) of rank ``rank`` when ``heads`` heads are split as evenly as possible over
    ``world`` ranks (the first heads % world ranks take one more)."""
    base, extra = divmod(heads, world)
    n = base + (1 if rank < extra else 0)
    return rank * base + min(rank, extra), n


def token_ranges(tokens: int, world: int) -> list[int]:
    """Token counts of the ranks' ranges when ``tokens`` tokens are split as evenly as possible."""
    base, extra = divmod(tokens, world)
    return [base + (1 if r < extra else 0) for r in range(world)]


class CudaIpc:
    """Peer mappings through the library's CUDA IPC calls."""

    export = staticmethod(lvsa_ipc_export)
    open = staticmethod(lvsa_ipc_import)
    close = staticmethod(lvsa_ipc_release)


class SequenceParallelAttention:
    """LVSA attention for one rank of a sequence-parallel group (see the module docstring).

    T, tokens_per_frame, heads, d, batch: the sizes of the whole call.  group: a torch.distributed process
    group of the ranks (one per GPU of a node), or None for the default group / a single process.
    chunk_tokens: token count of every rank's range (default: an even split).  ipc: the mapping layer
    (tests pass a stand-in).
    """

    def __init__(self, T: int, tokens_per_frame: int, heads: int, d: int, batch: int = 1, group=None,
                 chunk_tokens=None, device=None, ipc=None):
        import torch
        import torch.distributed as dist

        self.group = group
        distributed = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size(group) if distributed else 1
        self.rank = dist.get_rank(group) if distributed else 0
        self.T, self.P, self.heads, self.d, self.batch = T, tokens_per_frame, heads, d, batch
        tokens = T * tokens_per_frame
        self.chunk_tokens = [int(n) for n in (chunk_tokens if chunk_tokens is not None
                                              else token_ranges(tokens, self.world))]
        if len(self.chunk_tokens) != self.world or min(self.chunk_tokens) < 0 or sum(self.chunk_tokens) != tokens:
            raise ValueError(f"chunk_tokens must give one count >= 0 per rank ({self.world}) summing to {tokens}")
        self.starts = [sum(self.chunk_tokens[:r]) for r in range(self.world + 1)]
        self.head0, self.band = head_band(self.rank, self.world, heads)
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        n = self.chunk_tokens[self.rank]

        def alloc(shape):
            return torch.empty(shape, dtype=torch.bfloat16, device=self.device)

        self.q, self.k, self.v, self.out = (alloc((batch, n, heads, d)) for _ in range(4))
        if self.world == 1:
            self.q_band, self.k_band, self.v_band = self.q, self.k, self.v  # the whole sequence, every head
        elif self.band > 0:
            self.q_band, self.k_band, self.v_band = (alloc((batch, tokens, self.band, d)) for _ in range(3))
        else:
            self.q_band = self.k_band = self.v_band = None  # more ranks than heads: this rank only holds tokens
        self._lists_dev = None  # device copy of the lists for host_call
        self._ipc = ipc if ipc is not None else CudaIpc()
        self._opened = []
        own = [self.q, self.k, self.v, self.out]
        if self.world == 1:
            self.tables = [[t.data_ptr()] for t in own]
            return
        mine = [self._ipc.export(t) if n > 0 else None for t in own]
        everyone = [None] * self.world
        dist.all_gather_object(everyone, mine, group=group)
        self.tables = [[0] * self.world for _ in range(4)]
        try:
            for r in range(self.world):
                for x in range(4):
                    if r == self.rank:
                        self.tables[x][r] = own[x].data_ptr() if n > 0 else 0
                    elif self.chunk_tokens[r] > 0:
                        ptr = self._ipc.open(everyone[r][x])
                        self._opened.append(ptr)
                        self.tables[x][r] = ptr
        except Exception:
            self._unmap()
            raise

    def _barrier(self) -> None:
        import torch
        import torch.distributed as dist

        if self.device.type == "cuda":
            torch.cuda.current_stream(self.device).synchronize()
        dist.barrier(group=self.group)

    def __call__(self, lists, scale: float = 0.0, events: list | None = None):
        """One call: ``out`` <- attention of the whole sequence, for this rank's tokens and every head.
        lists: CUDA int32 [T, L] frame lists (the same on every rank).  events: if a list, a tuple of three
        CUDA events (before the gather, between gather and attention, after the attention) recorded on the
        current stream is appended to it."""
        import torch

        ev = None
        if events is not None:
            ev = tuple(torch.cuda.Event(enable_timing=True) for _ in range(3))
            events.append(ev)
        if self.world > 1:
            self._barrier()  # every rank's q, k, v written
        if ev:
            ev[0].record()
        if self.band > 0 and self.world > 1:
            lvsa_seq_to_heads(self.tables[0], self.tables[1], self.tables[2], self.chunk_tokens, self.head0,
                              self.band, self.q_band, self.k_band, self.v_band, heads=self.heads)
        if ev:
            ev[1].record()
        if self.band > 0:
            lvsa_attention_to_chunks(self.q_band, self.k_band, self.v_band, lists, self.P, self.tables[3],
                                     self.chunk_tokens, self.heads, self.head0, scale=scale)
        if ev:
            ev[2].record()
        if self.world > 1:
            self._barrier()  # every rank's output rows stored
        return self.out

    def host_call(self, q_host, k_host, v_host, lists_host, out_host, scale: float = 0.0):
        """One call on host buffers: this rank's token range of Q, K, V (CPU bf16 [batch, n, heads, d], pinned
        for asynchronous copies) in, its range of the output out.  lists_host: CPU int32 [T, L].  Asynchronous
        on the current stream: synchronise before reading out_host.

        With one rank the whole call is ``lvsa_attention_host``: uploads and readback pipelined against the
        kernel by bands of heads, staged in this object's buffers.  With several ranks the range buffers must be
        complete on every rank before any rank gathers, so the copies go before and after the call."""
        import torch

        if self._lists_dev is None or tuple(self._lists_dev.shape) != tuple(lists_host.shape):
            self._lists_dev = torch.empty(tuple(lists_host.shape), dtype=torch.int32, device=self.device)
        if self.world == 1:
            return lvsa_attention_host(q_host, k_host, v_host, lists_host, self.P, out_host, self.q, self.k, self.v,
                                       self._lists_dev, self.out, scale=scale)
        for dev, host in ((self.q, q_host), (self.k, k_host), (self.v, v_host), (self._lists_dev, lists_host)):
            dev.copy_(host, non_blocking=True)
        self(self._lists_dev, scale=scale)
        out_host.copy_(self.out, non_blocking=True)
        return out_host

    def _unmap(self) -> None:
        while self._opened:
            self._ipc.close(self._opened.pop())

    def close(self) -> None:
        """Unmaps the peers' buffers; every rank calls it before any rank frees its own."""
        self._unmap()
        if self.world > 1:
            self._barrier()
