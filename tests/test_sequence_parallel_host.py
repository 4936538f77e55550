"""Host logic of the sequence-parallel (Ulysses-layout) call, without a GPU: the split of tokens and heads
over the ranks, and the exchange of buffer handles between two gloo ranks (with a stand-in for the CUDA IPC
layer, on CPU tensors)."""

import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_token_ranges_and_head_bands_partition_the_call(lib):
    from block_sparse_attention_frame_b200.sequence_parallel import head_band, token_ranges

    for tokens in (1, 7, 512, 188760):
        for world in range(1, 9):
            n = token_ranges(tokens, world)
            assert len(n) == world and sum(n) == tokens and max(n) - min(n) <= 1
    for heads in range(1, 41):
        for world in range(1, 9):
            bands = [head_band(r, world, heads) for r in range(world)]
            assert [h for h0, k in bands for h in range(h0, h0 + k)] == list(range(heads))


def test_single_process_is_the_plain_call_layout(lib):
    from block_sparse_attention_frame_b200.sequence_parallel import SequenceParallelAttention

    sp = SequenceParallelAttention(4, 16, 3, 64, batch=2, device="cpu")
    assert sp.world == 1 and sp.chunk_tokens == [64] and sp.starts == [0, 64]
    assert (sp.head0, sp.band) == (0, 3)
    assert tuple(sp.q.shape) == (2, 64, 3, 64) and sp.q_band is sp.q  # nothing to gather
    assert sp.tables[3] == [sp.out.data_ptr()]
    with pytest.raises(ValueError):
        SequenceParallelAttention(4, 16, 3, 64, chunk_tokens=[60], device="cpu")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


WORKER = r"""
import os, sys, datetime
sys.path.insert(0, {root!r})
import torch.distributed as dist
from block_sparse_attention_frame_b200.sequence_parallel import SequenceParallelAttention

rank = int(os.environ["RANK"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
opened, closed = [], []


class FakeIpc:
    # a handle names the exporting rank and its address; "mapping" it gives a distinct fake address
    def export(self, t):
        return ("%d:%d" % (rank, t.data_ptr())).encode()

    def open(self, handle):
        r, p = handle.decode().split(":")
        opened.append(int(p))
        return (int(r) + 1) * 10**15 + int(p)

    def close(self, ptr):
        closed.append(ptr)


chunks = [700, 0, 500] if {world} == 3 else [700, 500]
sp = SequenceParallelAttention(4, 300, 5, 64, batch=1, chunk_tokens=chunks, device="cpu", ipc=FakeIpc())
own = [t.data_ptr() if t.numel() else 0 for t in (sp.q, sp.k, sp.v, sp.out)]
everyone = [None] * {world}
dist.all_gather_object(everyone, own)
for x in range(4):
    for r in range({world}):
        want = own[x] if r == rank else ((r + 1) * 10**15 + everyone[r][x] if chunks[r] else 0)
        assert sp.tables[x][r] == want, (x, r, sp.tables[x][r], want)
assert sp.starts == [sum(chunks[:r]) for r in range({world} + 1)]
assert tuple(sp.q.shape) == (1, chunks[rank], 5, 64)
bands = [None] * {world}
dist.all_gather_object(bands, (sp.head0, sp.band))
assert [h for h0, n in bands for h in range(h0, h0 + n)] == list(range(5))
if sp.band:
    assert tuple(sp.q_band.shape) == (1, 1200, sp.band, 64)
n_peers = sum(1 for r in range({world}) if r != rank and chunks[r])
assert len(opened) == 4 * n_peers
sp.close()
assert sorted(closed) == sorted((r + 1) * 10**15 + everyone[r][x] for r in range({world}) if r != rank and chunks[r]
                                for x in range(4))
dist.destroy_process_group()
print("RESULT", rank, "ok", flush=True)
"""


@pytest.mark.parametrize("world", [2, 3])
def test_handle_exchange_over_gloo_ranks(tmp_path, lib, world):
    port = _free_port()
    script = tmp_path / "worker.py"
    script.write_text(WORKER.format(root=ROOT, world=world))
    procs = []
    for rank in range(world):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.STDOUT, text=True))
    outs = []
    for p in procs:
        try:
            outs.append(p.communicate(timeout=180)[0])
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            raise
    for rank, (p, out) in enumerate(zip(procs, outs)):
        assert p.returncode == 0, out
        assert f"RESULT {rank} ok" in out, out
