"""GPU parity: the CUDA path (C-ABI list builder + sm_100a kernel, called through
the C ABI) against the fp64 oracle, element by element.

Tolerance (stated for unit-variance bf16 inputs with fp32 accumulation):
max-abs error <= 2e-2 and mean-abs error <= 2e-3 against the oracle run in
float64 on the same bf16-rounded inputs.
"""

import numpy as np
import pytest
import torch

from oracle import attention as OA
from oracle import lists as OL

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
# mean-abs error relative to the mean output magnitude at full sizes: bf16 rounding of the output alone is
# ~0.2 % on average, P rounded to bf16 adds a similar random share
REL_MEAN = 1e-2


def run_kernel(lib, q, k, v, lists_np, P, scale=0.0):
    lists = torch.from_numpy(np.ascontiguousarray(lists_np, dtype=np.int32)).cuda()
    out = lib.lvsa_attention(q, k, v, lists, P, scale=scale)
    torch.cuda.synchronize()
    return out


def errors(got, ref):
    err = np.abs(got.astype(np.float64) - ref)
    return float(err.max()), float(err.mean())


def assert_close(got, ref, what=""):
    mx, mean = errors(got, ref)
    assert np.isfinite(got).all(), what
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max-abs {mx:.3e} mean-abs {mean:.3e}"
    return mx, mean


def make(T, P, H, d, B=1, seed=0, correlated=True):
    import synthetic

    return synthetic.make_custom(T, P, H, d, B=B, seed=seed, device="cuda", frame_correlated_k=correlated)


def host(*xs):
    """Host copies of the inputs for the oracle (it takes host tensors only)."""
    return [x.cpu() for x in xs]


def full_out(out):
    return out.float().cpu().numpy()


def test_tiny_workload_all_steps(gpu_lib):
    import synthetic

    w = synthetic.WORKLOADS["tiny"]
    q32, k32, v32 = synthetic.make_qkv(w, device="cpu", dtype=torch.float32)
    q, k, v = (x.to(torch.bfloat16) for x in (q32, k32, v32))
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    for s in range(w.steps):
        lists = gpu_lib.lvsa_build_frame_lists(w.T, w.C, w.W, s)
        out = full_out(run_kernel(gpu_lib, qd, kd, vd, lists, w.P))
        ref = OA.sparse_attention(q, k, v, OL.frame_lists(w.T, w.C, w.W, s), w.P)
        assert_close(out, ref, f"tiny step {s}")
        # also within tolerance of the unrounded fp32 draws
        ref32 = OA.sparse_attention(q32, k32, v32, OL.frame_lists(w.T, w.C, w.W, s), w.P)
        assert errors(out, ref32)[0] <= 5e-2


def test_negative_control_wrong_step_fails(gpu_lib):
    import synthetic

    w = synthetic.WORKLOADS["tiny"]
    q, k, v = synthetic.make_qkv(w, device="cpu")
    out = full_out(run_kernel(gpu_lib, q.cuda(), k.cuda(), v.cuda(), gpu_lib.lvsa_build_frame_lists(8, 4, 2, 0),
                              w.P))
    ref_wrong = OA.sparse_attention(q, k, v, OL.frame_lists(8, 4, 2, 1), w.P)
    mx, mean = errors(out, ref_wrong)
    assert mx > MAX_ABS and mean > MEAN_ABS


@pytest.mark.parametrize("T,P,H,d,B,C,W,s", [
    (6, 200, 3, 128, 2, 3, 1, 4),     # 2 query tiles per frame (128 + 72 rows), ragged K/V runs
    (7, 300, 2, 64, 1, 4, 2, 3),      # d = 64, 3 query tiles (128+128+44)
    (10, 129, 2, 128, 1, 5, 2, 7),    # one-row tail tiles everywhere
    (5, 17, 4, 128, 1, 2, 1, 1),      # tokens per frame below one tile
    (9, 256, 1, 128, 1, 9, 3, 0),     # C = T: dense
    (12, 96, 2, 128, 1, 5, 5, 2),     # G = 0: pure sliding window
    (1, 1000, 2, 128, 1, 21, 9, 0),   # T = 1
    (5, 300, 2, 128, 2, 3, 1, 2),     # batch 2, 256-row blocks straddling frame boundaries
    (6, 700, 3, 64, 2, 3, 2, 5),      # batch 2, d = 64, straddling blocks
    (7, 1, 2, 64, 1, 3, 1, 4),        # one token per frame
    (4, 2, 1, 128, 3, 2, 2, 1),       # two tokens per frame, batch 3
    (9, 130, 1, 128, 1, 1, 1, 0),     # C = W = 1: every frame attends only itself
    (12, 520, 2, 128, 1, 6, 2, 5),    # P % 8 == 0: tiles span two runs (8 tokens of one, 120 of the next)
    (12, 40, 2, 64, 2, 6, 2, 7),      # P % 8 == 0, frames shorter than a tile: packed tiles stay partial
    (9, 1560, 1, 128, 1, 5, 2, 3),    # the 24-token frame tails packed with the next run
])
def test_ragged_shapes_full_parity(gpu_lib, T, P, H, d, B, C, W, s):
    q, k, v = make(T, P, H, d, B=B, seed=T * 1000 + P)
    lists = gpu_lib.lvsa_build_frame_lists(T, C, W, s)
    out = full_out(run_kernel(gpu_lib, q, k, v, lists, P))
    ref = OA.sparse_attention(*host(q, k, v), OL.frame_lists(T, C, W, s), P)
    assert_close(out, ref, f"T={T} P={P} d={d}")


def test_dense_lists_equal_full_attention(gpu_lib):
    T, P, H, d = 4, 160, 2, 128
    q, k, v = make(T, P, H, d, seed=77)
    out = full_out(run_kernel(gpu_lib, q, k, v, gpu_lib.lvsa_build_frame_lists(T, T, 1, 0), P))
    assert_close(out, OA.dense_attention(*host(q, k, v)), "dense")


def test_explicit_scale(gpu_lib):
    T, P, H, d = 5, 130, 2, 64
    q, k, v = make(T, P, H, d, seed=5)
    lists = gpu_lib.lvsa_build_frame_lists(T, 3, 1, 2)
    out = full_out(run_kernel(gpu_lib, q, k, v, lists, P, scale=0.05))
    assert_close(out, OA.sparse_attention(*host(q, k, v), OL.frame_lists(T, 3, 1, 2), P, scale=0.05), "scale")


def test_large_logits_rescale_path(gpu_lib):
    # keys growing along the list order force many running-max updates (O rescales)
    T, P, H, d = 6, 256, 1, 128
    q, k, v = make(T, P, H, d, seed=8)
    ramp = torch.linspace(0, 6, T * P, device="cuda").view(1, T * P, 1, 1)
    k = (k.float() + ramp * q.float().mean(dim=1, keepdim=True)).to(torch.bfloat16).contiguous()
    q = (q.float() * 2).to(torch.bfloat16).contiguous()
    lists = gpu_lib.lvsa_build_frame_lists(T, 4, 2, 3)
    out = full_out(run_kernel(gpu_lib, q, k, v, lists, P))
    assert_close(out, OA.sparse_attention(*host(q, k, v), OL.frame_lists(T, 4, 2, 3), P), "rescale")


@pytest.mark.parametrize("key_pos", [5, 40, 70, 127])
def test_max_jump_inside_a_later_tile(gpu_lib, key_pos):
    """One key far above everything before it, at position key_pos of a later full tile: for key_pos < 64 the
    speculative softmax sees it only through the row sum of keys 0..63, for key_pos >= 64 through the max of
    keys 64..127.  Either way the rows must rescale and match the oracle."""
    T, P, H, d = 4, 512, 1, 128
    q, k, v = make(T, P, H, d, seed=90 + key_pos)
    lists = gpu_lib.lvsa_build_frame_lists(T, T, 1, 0)  # dense: one run of 16 full tiles
    qf, kf = q.float(), k.float()
    tok = 5 * 128 + key_pos  # a key in the sixth tile of the walk
    u = torch.randn(d, generator=torch.Generator().manual_seed(key_pos)).to(qf.device)
    u = u / u.norm()
    kf[0, tok, 0, :] = 40.0 * u  # far along a direction that the queries of frame 0 share
    qf[0, :P, 0, :] += 4.0 * u
    q, k = qf.to(torch.bfloat16).contiguous(), kf.to(torch.bfloat16).contiguous()
    out = full_out(run_kernel(gpu_lib, q, k, v, lists, P))
    ref = OA.sparse_attention(*host(q, k, v), OL.frame_lists(T, T, 1, 0), P)
    # the key dominates the rows of frame 0: its logit is far above the rest
    S = (q.float()[0, :P, 0, :] @ k.float()[0, :, 0, :].T) / np.sqrt(d)
    gap = (S[:, tok] - S[:, :tok].max(dim=1).values).median().item() * 1.4427
    assert gap > 8, gap
    assert_close(out, ref, f"max jump at key {key_pos}")


def test_unsorted_lists_same_result(gpu_lib):
    T, P, H, d = 8, 150, 2, 128
    q, k, v = make(T, P, H, d, seed=3)
    lists = gpu_lib.lvsa_build_frame_lists(T, 4, 2, 5)
    rev = np.ascontiguousarray(lists[:, ::-1])
    a = full_out(run_kernel(gpu_lib, q, k, v, lists, P))
    b = full_out(run_kernel(gpu_lib, q, k, v, rev, P))
    assert_close(b, a.astype(np.float64), "list order")


def test_bad_list_entry_flagged_and_skipped(gpu_lib):
    T, P, H, d = 6, 64, 1, 64
    q, k, v = make(T, P, H, d, seed=4)
    gpu_lib.lvsa_get_device_status(clear=True)
    lists = gpu_lib.lvsa_build_frame_lists(T, 3, 1, 0).copy()
    good = [list(r) for r in lists]
    lists[2, 1] = 99  # out of range: skipped, status bit set
    good[2] = [f for j, f in enumerate(good[2]) if j != 1]
    out = full_out(run_kernel(gpu_lib, q, k, v, lists, P))
    assert gpu_lib.lvsa_get_device_status(clear=True) & gpu_lib.LVSA_DEV_BAD_LIST
    assert_close(out, OA.sparse_attention(*host(q, k, v), good, P), "bad list")


def test_watchdog_times_out_and_context_survives(gpu_lib):
    gpu_lib.lvsa_get_device_status(clear=True)
    gpu_lib.lvsa_watchdog_selftest(2_000_000)  # 2 ms budget on a barrier nobody arrives on
    torch.cuda.synchronize()
    assert gpu_lib.lvsa_get_device_status(clear=True) & gpu_lib.LVSA_DEV_TIMEOUT
    # the context is still usable
    test_dense_lists_equal_full_attention(gpu_lib)
    assert gpu_lib.lvsa_get_device_status(clear=True) == 0


def sample_rows(T, P, seed, per_frame=40):
    g = np.random.default_rng(seed)
    frames = sorted(set([0, 1, T // 2, T - 2, T - 1] + list(g.choice(T, 3, replace=False))))
    # rows 0, 1, 127, 128 and the last 25 rows of the frame (its 24-row tail past the last full 128-row
    # tile at P = 1560, and the row before it)
    base = sorted(set([0, 1, 127, 128] + list(range(max(0, P - 25), P))))
    rows = []
    for f in frames:
        extra = g.choice(P, max(0, per_frame - len(base)), replace=False)
        rows += [f * P + r for r in sorted(set(base) | set(int(x) for x in extra))]
    return rows


@pytest.mark.parametrize("name,steps", [
    ("wan1.3b_1x", [0]),
    ("wan1.3b_6x", [0, 17, 49]),
    ("hunyuan1.5_1.5x", [0, 2, 31]),
    ("hunyuan1.5_2x", [0, 40]),
    ("wan14b_6x", [5]),
])
def test_full_size_workloads_sampled_rows(gpu_lib, name, steps):
    import synthetic

    w = synthetic.WORKLOADS[name]
    q, k, v = synthetic.make_qkv(w, device="cuda")
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    # the first step: 128 rows in each of 8 frames (frames 0, 1, T/2, T-2, T-1 and 3 seeded ones; rows 0, 1,
    # 127, 128 and the frame's last 25, the rest seeded); later steps: 40 per frame
    rows_first = sample_rows(w.T, w.P, seed=w.seed, per_frame=128)
    rows_later = sample_rows(w.T, w.P, seed=w.seed)
    for i, s in enumerate(steps):
        rows = rows_first if i == 0 else rows_later
        lists = gpu_lib.lvsa_build_frame_lists(w.T, w.C, w.W, s)
        out = run_kernel(gpu_lib, q, k, v, lists, w.P)
        got = out[:, rows].float().cpu().numpy()
        ref = OA.sparse_attention_rows(qc, kc, vc, OL.frame_lists(w.T, w.C, w.W, s), w.P, rows)
        assert_close(got, ref, f"{name} step {s}")
        # the outputs are small at these sizes (RMS ~0.01), so the absolute bound is loose: also bound the
        # error relative to the mean output magnitude, and check that the lists of step s+1 (anchors moved
        # by one frame) fail it by far (negative control)
        rel = float(np.abs(got - ref).mean() / np.abs(ref).mean())
        assert rel <= REL_MEAN, f"{name} step {s}: relative mean error {rel:.3e}"
        if i == 0:
            wrong = OA.sparse_attention_rows(qc, kc, vc, OL.frame_lists(w.T, w.C, w.W, s + 1), w.P, rows)
            rel_wrong = float(np.abs(got - wrong).mean() / np.abs(wrong).mean())
            print(f"{name} step {s}: relative mean error {rel:.3e}, against step {s + 1}'s lists {rel_wrong:.3e}")
            if w.C < w.T:
                assert rel_wrong > 10 * REL_MEAN, f"negative control {name}: {rel_wrong:.3e}"
        assert torch.isfinite(out).all()
        del out
    torch.cuda.empty_cache()


@pytest.mark.parametrize("T,P,d", [(10, 300, 128), (6, 200, 64), (9, 517, 128)])
def test_random_lists_are_sets(gpu_lib, T, P, d):
    # arbitrary per-frame lists, unsorted and with duplicates: each row is the set of its
    # frames; query blocks that straddle two frames attend the union with per-row masks
    g = np.random.default_rng(T * P)
    L = 5
    lists = g.integers(0, T, size=(T, L)).astype(np.int32)
    lists[1, :] = lists[1, 0]                    # one frame listed L times
    q, k, v = make(T, P, 2, d, seed=P)
    out = full_out(run_kernel(gpu_lib, q, k, v, lists, P))
    ref = OA.sparse_attention(*host(q, k, v), [sorted(set(int(f) for f in r)) for r in lists], P)
    assert_close(out, ref, "random set lists")


def test_frame_without_valid_entries_gives_zeros(gpu_lib):
    T, P, H, d = 7, 300, 2, 128
    q, k, v = make(T, P, H, d, seed=21)
    gpu_lib.lvsa_get_device_status(clear=True)
    lists = gpu_lib.lvsa_build_frame_lists(T, 3, 1, 1).copy()
    lists[4, :] = -1
    out = full_out(run_kernel(gpu_lib, q, k, v, lists, P))
    assert gpu_lib.lvsa_get_device_status(clear=True) & gpu_lib.LVSA_DEV_BAD_LIST
    assert np.all(out[:, 4 * P:5 * P] == 0)
    good = [list(r) for r in lists]
    rows = [r for r in range(T * P) if r // P != 4]
    ref = OA.sparse_attention_rows(*host(q, k, v), good, P, rows)
    assert_close(out[:, rows], ref, "other frames")


@pytest.mark.parametrize("T,P,d", [(4, 512, 128), (5, 100, 64)])
def test_blocks_with_no_listed_frame_write_zeros(gpu_lib, T, P, d):
    """Query blocks that lie wholly inside a frame with no valid list entry walk no K/V tile at all: their
    rows are still written, as zeros, whatever the output buffer held (P = 512: 256-row blocks aligned to
    the frames; P = 100: one block per frame)."""
    q, k, v = make(T, P, 2, d, seed=17)
    gpu_lib.lvsa_get_device_status(clear=True)
    lists = gpu_lib.lvsa_build_frame_lists(T, 3, 1, 2).copy()
    lists[1, :] = -1
    out = torch.full_like(q, float("nan"))
    gpu_lib.lvsa_attention(q, k, v, torch.from_numpy(lists).cuda(), P, out=out)
    torch.cuda.synchronize()
    assert gpu_lib.lvsa_get_device_status(clear=True) & gpu_lib.LVSA_DEV_BAD_LIST
    got = full_out(out)
    assert np.all(got[:, P:2 * P] == 0)
    rows = [r for r in range(T * P) if r // P != 1]
    ref = OA.sparse_attention_rows(*host(q, k, v), [list(r) for r in lists], P, rows)
    assert_close(got[:, rows], ref, "other frames")


def run_host_path(lib, q, k, v, lists_np, P, heads_per_band=0, scale=0.0, stale=None):
    """The host-buffer entry point: CPU tensors in, CPU tensor out, staging buffers on the GPU.  `stale`:
    a value the staging buffers hold before the call (a row the kernel reads but the call did not upload
    would leak it into the output)."""
    qh, kh, vh = (x.cpu().contiguous().pin_memory() for x in (q, k, v))
    lh = torch.from_numpy(np.ascontiguousarray(lists_np, dtype=np.int32))
    oh = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
    qd, kd, vd, od = (torch.empty(qh.shape, dtype=torch.bfloat16, device="cuda") for _ in range(4))
    if stale is not None:
        for x in (qd, kd, vd, od):
            x.fill_(stale)
    ld = torch.empty(lh.shape, dtype=torch.int32, device="cuda")
    lib.lvsa_attention_host(qh, kh, vh, lh, P, oh, qd, kd, vd, ld, od, scale=scale, heads_per_band=heads_per_band)
    torch.cuda.synchronize()
    return oh


@pytest.mark.parametrize("T,P,H,d,B,C,W,s,hb", [
    (8, 64, 2, 64, 1, 4, 2, 1, 1),      # tiny shape, one head per band
    (8, 64, 2, 64, 1, 4, 2, 1, 0),      # automatic bands
    (6, 300, 3, 128, 2, 3, 1, 4, 2),    # straddling query blocks, batch 2, uneven bands (2 + 1 heads)
    (5, 96, 5, 64, 1, 5, 2, 0, 3),      # dense lists, ragged frames, bands of 3 + 2
    # batch 1, 256-row blocks: the first band's Q goes up, and the last band's output comes back, in pieces
    (10, 300, 3, 128, 1, 5, 2, 3, 1),   # three bands: first and last in pieces
    (10, 300, 2, 128, 1, 5, 2, 3, 1),   # two bands
    (10, 300, 3, 128, 1, 5, 2, 3, 3),   # one band, both in pieces
])
def test_host_buffer_path_equals_device_path(gpu_lib, T, P, H, d, B, C, W, s, hb):
    q, k, v = make(T, P, H, d, B=B, seed=11)
    lists = gpu_lib.lvsa_build_frame_lists(T, C, W, s)
    dev_out = run_kernel(gpu_lib, q, k, v, lists, P).cpu()
    # staging buffers full of NaN: every row the kernel reads must have been uploaded by the call
    host_out = run_host_path(gpu_lib, q, k, v, lists, P, heads_per_band=hb, stale=float("nan"))
    # same kernel on the same bf16 inputs, one band of heads at a time: identical bits
    assert torch.equal(host_out.view(torch.int16), dev_out.view(torch.int16))
    ref = OA.sparse_attention(*host(q, k, v), OL.frame_lists(T, C, W, s), P)
    assert_close(host_out.float().numpy(), ref, "host-buffer path")


@pytest.mark.parametrize("H,hb", [(3, 1), (2, 2)])
def test_host_buffer_path_hand_made_lists(gpu_lib, H, hb):
    """Lists made by hand (unsorted, a repeated entry, frames almost nobody lists, runs ending inside a
    tile), staging buffers full of NaN: every row the kernel reads comes from the call's own uploads, and the
    result is the device call's, bit for bit."""
    T, P, d = 12, 520, 128
    rows = []
    for t in range(T):
        rows.append([(t + 5) % T, t, 9 if t < 6 else 2, t])  # frame 9 or 2 for every row; 10, 11 mostly unread
    lists = np.array(rows, dtype=np.int32)
    q, k, v = make(T, P, H, d, seed=31)
    dev_out = run_kernel(gpu_lib, q, k, v, lists, P).cpu()
    host_out = run_host_path(gpu_lib, q, k, v, lists, P, heads_per_band=hb, stale=float("nan"))
    assert torch.isfinite(host_out.float()).all()
    assert torch.equal(host_out.view(torch.int16), dev_out.view(torch.int16))
    ref = OA.sparse_attention(*host(q, k, v), [sorted(set(r)) for r in rows], P)
    assert_close(host_out.float().numpy(), ref, "host-buffer path, hand-made lists")


def test_host_buffer_path_full_size_heads(gpu_lib):
    """Wan-1.3B 1x shape (T=21, P=1560, 12 heads): automatic bands, bit-identical to the device path."""
    q, k, v = make(21, 1560, 12, 128, seed=5)
    lists = gpu_lib.lvsa_build_frame_lists(21, 21, 9, 0)
    dev_out = run_kernel(gpu_lib, q, k, v, lists, 1560).cpu()
    host_out = run_host_path(gpu_lib, q, k, v, lists, 1560)
    assert torch.equal(host_out.view(torch.int16), dev_out.view(torch.int16))


def test_host_buffer_path_pageable_memory(gpu_lib):
    """Pageable (not pinned) host tensors: the copies stall instead of overlapping, the result is the same."""
    T, P, H, d = 6, 200, 3, 64
    q, k, v = make(T, P, H, d, seed=21)
    lists = gpu_lib.lvsa_build_frame_lists(T, 4, 2, 2)
    dev_out = run_kernel(gpu_lib, q, k, v, lists, P).cpu()
    qh, kh, vh = (x.cpu().contiguous() for x in (q, k, v))
    oh = torch.empty(qh.shape, dtype=torch.bfloat16)
    qd, kd, vd, od = (torch.empty(qh.shape, dtype=torch.bfloat16, device="cuda") for _ in range(4))
    ld = torch.empty(lists.shape, dtype=torch.int32, device="cuda")
    gpu_lib.lvsa_attention_host(qh, kh, vh, torch.from_numpy(lists), P, oh, qd, kd, vd, ld, od)
    torch.cuda.synchronize()
    assert torch.equal(oh.view(torch.int16), dev_out.view(torch.int16))


@pytest.mark.parametrize("P,d", [(16, 64), (40, 128)])
def test_maximum_frame_count(gpu_lib, P, d):
    """T = 4096, the largest frame count the kernel's frame bitmaps cover: sampled rows against the oracle,
    including the first and last frames (anchors wrap around the end of the sequence)."""
    T, C, W, s = 4096, 7, 3, 4093
    q, k, v = make(T, P, 1, d, seed=31)
    lists = gpu_lib.lvsa_build_frame_lists(T, C, W, s)
    out = run_kernel(gpu_lib, q, k, v, lists, P)
    g = np.random.default_rng(5)
    frames = sorted(set([0, 1, 2047, 4094, 4095] + list(g.choice(T, 5, replace=False))))
    rows = [f * P + r for f in frames for r in range(P)]
    got = out[:, rows].float().cpu().numpy()
    ref = OA.sparse_attention_rows(*host(q, k, v), OL.frame_lists(T, C, W, s), P, rows)
    assert_close(got, ref, f"T=4096 P={P} d={d}")
    assert torch.isfinite(out).all()


def test_bench_json_line_contract():
    """bench.py on the tiny workload prints one JSON line with every key of the benchmark contract."""
    import json
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--workload", "tiny", "--steps", "3",
                          "--warmup", "3", "--no-cpu-baseline"], capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == 3 and d["warmup"] >= 3 and d["value"] > 0
    assert d["config"]["workload"] == "tiny"
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in d["roofline"], key
    for key in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"):
        assert key in d["e2e"], key
    assert d["e2e"]["h2d_bytes_per_step"] > 0 and d["e2e"]["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] == 3
    for key in ("sm_mhz", "sm_max_mhz", "reasons"):
        assert key in d["clocks"], key


def test_cuda_graph_capture_and_replay(gpu_lib):
    """Both entry points can be captured into a CUDA graph (tensor maps travel by value in the launch
    parameters; the host-buffer call's internal streams join the capture through its events); replays
    give the eager results bit for bit, also after the inputs are changed in place."""
    T, P, H, d = 6, 300, 3, 128
    q, k, v = make(T, P, H, d, seed=41)
    lists_np = gpu_lib.lvsa_build_frame_lists(T, 4, 2, 3)
    lists = torch.from_numpy(lists_np).cuda()
    out = torch.empty_like(q)
    qh, kh, vh = (x.cpu().contiguous().pin_memory() for x in (q, k, v))
    lh = torch.from_numpy(lists_np).pin_memory()
    oh = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
    stage = [torch.empty_like(q) for _ in range(4)]
    ld = torch.empty_like(lists)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up outside the capture (first-call setup)
        gpu_lib.lvsa_attention(q, k, v, lists, P, out=out)
        gpu_lib.lvsa_attention_host(qh, kh, vh, lh, P, oh, stage[0], stage[1], stage[2], ld, stage[3])
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g1, g2 = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g1):
        gpu_lib.lvsa_attention(q, k, v, lists, P, out=out)
    with torch.cuda.graph(g2):
        gpu_lib.lvsa_attention_host(qh, kh, vh, lh, P, oh, stage[0], stage[1], stage[2], ld, stage[3])
    for trial in range(2):
        if trial == 1:  # new inputs in the same buffers
            q2, k2, v2 = make(T, P, H, d, seed=42)
            q.copy_(q2), k.copy_(k2), v.copy_(v2)
            qh.copy_(q2.cpu()), kh.copy_(k2.cpu()), vh.copy_(v2.cpu())
        out.zero_()
        oh.zero_()
        torch.cuda.synchronize()
        g1.replay()
        g2.replay()
        torch.cuda.synchronize()
        eager = gpu_lib.lvsa_attention(q, k, v, lists, P)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
        assert torch.equal(oh.view(torch.int16), eager.cpu().view(torch.int16))


def test_captured_host_call_follows_the_lists_at_replay(gpu_lib):
    """A captured host-buffer call reads the host lists at replay: captured with the lists of step 3,
    replayed after the host buffer was given those of step 4 (and the staging buffers filled with NaN), it
    gives the eager result for step 4, bit for bit -- one graph serves every denoising step."""
    T, P, H, d = 10, 300, 2, 128
    q, k, v = make(T, P, H, d, seed=43)
    qh, kh, vh = (x.cpu().contiguous().pin_memory() for x in (q, k, v))
    lh = torch.from_numpy(gpu_lib.lvsa_build_frame_lists(T, 5, 2, 3)).pin_memory()
    oh = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
    stage = [torch.empty_like(q) for _ in range(4)]
    ld = torch.empty(lh.shape, dtype=torch.int32, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # first-call setup outside the capture
        gpu_lib.lvsa_attention_host(qh, kh, vh, lh, P, oh, stage[0], stage[1], stage[2], ld, stage[3],
                                    heads_per_band=1)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        gpu_lib.lvsa_attention_host(qh, kh, vh, lh, P, oh, stage[0], stage[1], stage[2], ld, stage[3],
                                    heads_per_band=1)
    lists4 = gpu_lib.lvsa_build_frame_lists(T, 5, 2, 4)
    assert not np.array_equal(lists4, lh.numpy())
    lh.copy_(torch.from_numpy(lists4))
    for x in stage:
        x.fill_(float("nan"))
    oh.zero_()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    eager = run_kernel(gpu_lib, q, k, v, lists4, P).cpu()
    assert torch.equal(oh.view(torch.int16), eager.view(torch.int16))
