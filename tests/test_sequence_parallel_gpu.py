"""GPU parity of the sequence-parallel (Ulysses-layout) path: the band gather (lvsa_seq_to_heads) and the
attention with output rows routed to the token-range owners (lvsa_attention_to_chunks).

Ranks are emulated in one process (every "peer" buffer is a local tensor; the kernels of one rank never wait
on another's, so this is the same computation), and run for real as two or three processes sharing one GPU
through CUDA IPC mappings, ordered by a gloo process group.  The outputs must equal the single call (lvsa_attention
on the whole tensors) bit for bit: every head is computed by the same kernel on the same data, only the
buffers differ.  The single call itself is checked against the fp64 oracle in test_attention_gpu.py; the
tiny case is checked against the oracle here too.
"""

import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch

from oracle import attention as OA
from oracle import lists as OL

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def emulate(lib, q, k, v, lists, P, chunk_tokens):
    """Every rank of a len(chunk_tokens)-rank group, one after the other, on this GPU."""
    from block_sparse_attention_frame_b200.sequence_parallel import head_band

    B, ntok, H, d = q.shape
    N = len(chunk_tokens)
    starts = [sum(chunk_tokens[:r]) for r in range(N + 1)]
    qc, kc, vc = ([x[:, starts[r]:starts[r + 1]].contiguous() for r in range(N)] for x in (q, k, v))
    oc = [torch.full((B, n, H, d), float("nan"), dtype=torch.bfloat16, device=q.device) for n in chunk_tokens]
    for r in range(N):
        h0, band = head_band(r, N, H)
        if band == 0:
            continue
        qb, kb, vb = (torch.empty((B, ntok, band, d), dtype=torch.bfloat16, device=q.device) for _ in range(3))
        lib.lvsa_seq_to_heads(qc, kc, vc, chunk_tokens, h0, band, qb, kb, vb, heads=H)
        torch.cuda.synchronize()
        for x, xb in ((q, qb), (k, kb), (v, vb)):  # the gather is a pure copy of the band
            assert torch.equal(xb.view(torch.int16), x[:, :, h0:h0 + band].contiguous().view(torch.int16))
        lib.lvsa_attention_to_chunks(qb, kb, vb, lists, P, oc, chunk_tokens, H, h0)
    torch.cuda.synchronize()
    assert lib.lvsa_get_device_status(clear=True) == 0
    return torch.cat(oc, dim=1)


def same_bits(a, b):
    return torch.equal(a.contiguous().view(torch.int16), b.contiguous().view(torch.int16))


def test_tiny_workload_emulated_ranks_match_single_call_and_oracle(gpu_lib):
    import synthetic

    w = synthetic.WORKLOADS["tiny"]
    q, k, v = synthetic.make_qkv(w, device="cpu")
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    for s in (0, 5):
        lists_np = gpu_lib.lvsa_build_frame_lists(w.T, w.C, w.W, s)
        lists = torch.from_numpy(lists_np).cuda()
        ref = gpu_lib.lvsa_attention(qd, kd, vd, lists, w.P)
        torch.cuda.synchronize()
        oracle = OA.sparse_attention(q, k, v, OL.frame_lists(w.T, w.C, w.W, s), w.P)
        # 2 ranks (a head each), 3 ranks (one holds tokens but no head), uneven ranges with an empty one
        for chunks in ([256, 256], [100, 300, 112], [0, 512], [511, 0, 1]):
            out = emulate(gpu_lib, qd, kd, vd, lists, w.P, chunks)
            assert same_bits(out, ref), (s, chunks)
            err = np.abs(out.float().cpu().numpy() - oracle)
            assert err.max() <= 2e-2 and err.mean() <= 2e-3


@pytest.mark.parametrize("T,P,H,d,B,C,W,chunks", [
    (12, 300, 5, 128, 1, 5, 3, [1000, 0, 1700, 900]),   # 4 ranks: bands of 2, 1, 1, 1 heads
    (6, 256, 3, 128, 2, 4, 2, [512, 512, 512]),          # batch 2, frame-aligned ranges
    (7, 1560, 4, 128, 1, 4, 3, [2731, 2730, 2730, 2729]),  # video-sized frames, ranges across frame ends
    (9, 200, 2, 64, 1, 5, 2, [1, 1799]),                 # d = 64, a one-token range
])
def test_emulated_ranks_match_single_call(gpu_lib, T, P, H, d, B, C, W, chunks):
    import synthetic

    q, k, v = synthetic.make_custom(T, P, H, d, B=B, seed=T * 31 + H, device="cuda")
    lists = torch.from_numpy(gpu_lib.lvsa_build_frame_lists(T, C, W, 3)).cuda()
    ref = gpu_lib.lvsa_attention(q, k, v, lists, P)
    out = emulate(gpu_lib, q, k, v, lists, P, chunks)
    assert same_bits(out, ref)


def test_routed_call_writes_only_its_heads(gpu_lib):
    """Heads outside [head0, head0 + heads) of the output rows stay as they were."""
    import synthetic

    T, P, H, d = 5, 256, 4, 128
    q, k, v = synthetic.make_custom(T, P, H, d, seed=5, device="cuda")
    lists = torch.from_numpy(gpu_lib.lvsa_build_frame_lists(T, 3, 2, 1)).cuda()
    ref = gpu_lib.lvsa_attention(q, k, v, lists, P)
    chunks = [600, 680]
    outs = [torch.full((1, n, H, d), 7.0, dtype=torch.bfloat16, device="cuda") for n in chunks]
    qb, kb, vb = (x[:, :, 1:3].contiguous() for x in (q, k, v))
    gpu_lib.lvsa_attention_to_chunks(qb, kb, vb, lists, P, outs, chunks, H, 1)
    torch.cuda.synchronize()
    out = torch.cat(outs, dim=1)
    assert same_bits(out[:, :, 1:3], ref[:, :, 1:3])
    assert bool((out[:, :, 0] == 7.0).all()) and bool((out[:, :, 3] == 7.0).all())


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


WORKER = r"""
import os, sys, datetime
sys.path.insert(0, {root!r})
import torch
import torch.distributed as dist
import block_sparse_attention_frame_b200 as lvsa
import synthetic
from block_sparse_attention_frame_b200.sequence_parallel import SequenceParallelAttention

rank = int(os.environ["RANK"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
torch.cuda.set_device(0)
lvsa.lvsa_set_wait_budget_ns(500_000_000)
T, P, H, d = 10, 300, {heads}, 128
q, k, v = synthetic.make_custom(T, P, H, d, seed=77, device="cuda")
sp = SequenceParallelAttention(T, P, H, d, chunk_tokens={chunks}, device="cuda:0")
a, b = sp.starts[rank], sp.starts[rank + 1]
for dst, src in ((sp.q, q), (sp.k, k), (sp.v, v)):
    dst.copy_(src[:, a:b])
ok = True
for step in (0, 3, 4):
    lists = torch.from_numpy(lvsa.lvsa_build_frame_lists(T, 5, 3, step)).cuda()
    out = sp(lists)
    ref = lvsa.lvsa_attention(q, k, v, lists, P)
    torch.cuda.synchronize()
    ok = ok and torch.equal(out.view(torch.int16), ref[:, a:b].contiguous().view(torch.int16))
# the same call on host buffers: this rank's range in and out
qh, kh, vh = (x[:, a:b].cpu().contiguous().pin_memory() for x in (q, k, v))
for step in (1, 4):
    lists_np = lvsa.lvsa_build_frame_lists(T, 5, 3, step)
    oh = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
    sp.host_call(qh, kh, vh, torch.from_numpy(lists_np).pin_memory(), oh)
    torch.cuda.synchronize()
    ref = lvsa.lvsa_attention(q, k, v, torch.from_numpy(lists_np).cuda(), P)
    torch.cuda.synchronize()
    ok = ok and torch.equal(oh.view(torch.int16), ref[:, a:b].cpu().contiguous().view(torch.int16))
status = lvsa.lvsa_get_device_status(clear=True)
sp.close()
dist.destroy_process_group()
print("RESULT", rank, int(ok), status, flush=True)
"""


@pytest.mark.parametrize("world,heads,chunks", [
    (2, 3, [1300, 1700]),
    (3, 2, [1300, 0, 1700]),  # rank 1 holds no tokens, rank 2 no heads
])
def test_processes_share_one_gpu_through_ipc(tmp_path, gpu_lib, world, heads, chunks):
    """Ranks as processes on one GPU: each maps the others' buffers (lvsa_ipc_import), gathers its heads from
    them, and stores its output rows into them; each rank's output equals its rows of the single call, on
    device buffers and through host_call on host buffers.  Host barriers order the ranks; no kernel waits on
    another process."""
    port = _free_port()
    script = tmp_path / "worker.py"
    script.write_text(WORKER.format(root=ROOT, heads=heads, chunks=chunks))
    procs = []
    for rank in range(world):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.STDOUT, text=True))
    outs = []
    for p in procs:
        try:
            outs.append(p.communicate(timeout=300)[0])
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            raise
    for rank, (p, out) in enumerate(zip(procs, outs)):
        assert p.returncode == 0, out[-3000:]
        assert f"RESULT {rank} 1 0" in out, out[-3000:]


def test_bench_sequence_parallel_json_line():
    import json

    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "tiny", "--steps", "3",
                          "--warmup", "3", "--sequence-parallel"], capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["scaling"] == "strong" and d["n_gpus"] == 1 and d["value"] > 0
    assert "sequence-parallel" in d["config"]["parallelism"]
    assert d["e2e"]["h2d_bytes_per_step"] > 0 and d["gpu_launches"] == 3


def test_rows_routed_to_host_memory_take_the_system_scope_path(gpu_lib):
    """A range buffer that is not this GPU's memory (here pinned host memory, which the GPU addresses
    directly) makes the kernel release its stores at system scope, the path peer stores take; the rows
    written there equal the single call's."""
    import synthetic

    T, P, H, d = 6, 300, 2, 128
    q, k, v = synthetic.make_custom(T, P, H, d, seed=13, device="cuda")
    lists = torch.from_numpy(gpu_lib.lvsa_build_frame_lists(T, 4, 2, 3)).cuda()
    ref = gpu_lib.lvsa_attention(q, k, v, lists, P)
    chunks = [1000, 800]
    dev_part = torch.full((1, chunks[0], H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    host_part = torch.full((1, chunks[1], H, d), float("nan"), dtype=torch.bfloat16).pin_memory()
    gpu_lib.lvsa_attention_to_chunks(q, k, v, lists, P, [dev_part, host_part.data_ptr()], chunks, H, 0)
    torch.cuda.synchronize()
    assert gpu_lib.lvsa_get_device_status(clear=True) == 0
    assert same_bits(dev_part, ref[:, :chunks[0]])
    assert same_bits(host_part, ref[:, chunks[0]:].cpu())


def test_unaddressable_range_buffer_is_refused(gpu_lib):
    """Pageable host memory cannot be written by the GPU: the call returns an argument error before any
    launch."""
    import synthetic

    T, P, H, d = 4, 256, 1, 128
    q, k, v = synthetic.make_custom(T, P, H, d, seed=3, device="cuda")
    lists = torch.from_numpy(gpu_lib.lvsa_build_frame_lists(T, 3, 1, 0)).cuda()
    dev_part = torch.empty((1, 512, H, d), dtype=torch.bfloat16, device="cuda")
    pageable = torch.empty((1, 512, H, d), dtype=torch.bfloat16)  # not pinned
    with pytest.raises(gpu_lib.LvsaError) as e:
        gpu_lib.lvsa_attention_to_chunks(q, k, v, lists, P, [dev_part, pageable.data_ptr()], [512, 512], H, 0)
    assert e.value.status == gpu_lib.LVSA_ERR_INVALID_ARG


def test_unaddressable_source_range_is_refused(gpu_lib):
    """The gather reads every source range from the GPU: a pageable host buffer among them is refused with an
    argument error before any launch; the same range in pinned (mapped) host memory is read like any other."""
    T, P, H, d = 4, 256, 2, 128
    src = [torch.randn((1, 512, H, d), device="cuda").to(torch.bfloat16) for _ in range(3)]
    pageable = [torch.randn((1, 512, H, d)).to(torch.bfloat16) for _ in range(3)]
    bands = [torch.empty((1, 1024, 1, d), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    tables = [[s, p.data_ptr()] for s, p in zip(src, pageable)]
    with pytest.raises(gpu_lib.LvsaError) as e:
        gpu_lib.lvsa_seq_to_heads(*tables, [512, 512], 1, 1, *bands, heads=H)
    assert e.value.status == gpu_lib.LVSA_ERR_INVALID_ARG
    pinned = [p.pin_memory() for p in pageable]
    gpu_lib.lvsa_seq_to_heads(*[[s, p.data_ptr()] for s, p in zip(src, pinned)], [512, 512], 1, 1, *bands, heads=H)
    torch.cuda.synchronize()
    for b, s, p in zip(bands, src, pinned):
        want = torch.cat([s[:, :, 1:2], p.cuda()[:, :, 1:2]], dim=1)
        assert torch.equal(b.view(torch.int16), want.view(torch.int16))


def test_host_call_one_rank_equals_single_call(gpu_lib):
    """One rank: the host-buffer call of the sequence-parallel object (uploads and readback pipelined by bands of
    heads) gives the single call's output bit for bit."""
    import synthetic
    from block_sparse_attention_frame_b200.sequence_parallel import SequenceParallelAttention

    T, P, H, d, B = 6, 300, 3, 128, 2
    q, k, v = synthetic.make_custom(T, P, H, d, B=B, seed=61, device="cuda")
    lists_np = gpu_lib.lvsa_build_frame_lists(T, 3, 1, 4)
    ref = gpu_lib.lvsa_attention(q, k, v, torch.from_numpy(lists_np).cuda(), P)
    sp = SequenceParallelAttention(T, P, H, d, batch=B)
    qh, kh, vh = (x.cpu().pin_memory() for x in (q, k, v))
    oh = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
    for _ in range(2):  # the second call reuses the object's staging buffers
        oh.zero_()
        sp.host_call(qh, kh, vh, torch.from_numpy(lists_np).pin_memory(), oh)
        torch.cuda.synchronize()
        assert same_bits(oh, ref.cpu())
    sp.close()
