#!/usr/bin/env python
"""Benchmark of the LVSA sparse-attention hot path on B200.

One step = the whole per-denoising-step path for one synthetic batch:
build the frame lists of step s on the host (C ABI), upload them (pinned
memory, async on the stream), run the sm_100a sparse-attention kernel.  The
timed region holds exactly K steps (s = W..W+K-1 after W warm-up steps),
bracketed by a barrier and device synchronisation, timed with CUDA events on
the launching stream; for N > 1 the max over ranks is taken.  Inputs (Q, K, V,
O = 2.3 GB for the Wan-1.3B 6x workload) are larger than the 126 MB L2, so no
flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl lvsa|reference]

Prints one JSON line on rank 0.  ``--impl reference`` times the fp64 CPU
oracle (a bounded sample of the same workload per step) on the host cores.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-attn ms/call & effective TFLOP/s, T=121×1560 tok, 12 heads, d=128"
DEFAULT_WORKLOAD = "wan1.3b_6x"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def flops_per_call(w) -> float:
    """Selected blocks only: QK^T and PV, 2*P*(L*P)*d flops each per (b, h, t)."""
    return 4.0 * w.B * w.H * w.T * w.L * w.P * w.P * w.d


def algorithmic_bytes(w) -> float:
    """Q, K, V read once and O written once, bf16."""
    return 4.0 * w.B * w.T * w.P * w.H * w.d * 2


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        try:
            import torch

            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            sel = str(device_index)
        self.cmd = ["nvidia-smi", "-i", sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                    "-lms", "200"]

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), float(parts[2]), parts[3:]))
            except ValueError:
                continue
        if not rows:
            return None
        power = [r[2] for r in rows]
        busy = [r for r in rows if r[2] > 0.5 * max(power)] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in busy for i, v in enumerate(r[3][1:]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in busy), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(power), "samples": len(rows), "samples_under_load": len(busy),
                "reasons": reasons}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


ORACLE_KIND = ("oracle: fp64 numpy, one (head, query frame) at a time; its matrix products run in numpy's BLAS "
               "dgemm on `cores` threads")


def cpu_oracle_sample(w, seconds: float, seed: int = 0):
    """Time the fp64 oracle on whole (head, query-frame) units of the workload
    until ``seconds`` of CPU work are done.  Returns (flops, elapsed, units)."""
    import numpy as np
    import torch

    import synthetic
    from oracle import attention as OA
    from oracle import lists as OL

    # the sample needs the K/V tokens of the frames it touches only; draw the
    # workload's tensors on the CPU with a smaller head count to bound memory
    sub = synthetic.Workload(w.name + "-cpu-sample", T=w.T, P=w.P, H=1, d=w.d, C=w.C, W=w.W, seed=w.seed + 17)
    q, k, v = synthetic.make_qkv(sub, device="cpu")
    lists = OL.frame_lists(w.T, w.C, w.W, 0)
    g = np.random.default_rng(seed)
    frames = list(g.permutation(w.T))
    done = 0
    flops = 0.0
    t0 = time.perf_counter()
    for t in frames:
        rows = range(int(t) * w.P, (int(t) + 1) * w.P)
        OA.sparse_attention_rows(q, k, v, lists, w.P, rows)
        done += 1
        flops += 4.0 * w.P * (len(lists[int(t)]) * w.P) * w.d
        if time.perf_counter() - t0 >= seconds:
            break
    return flops, time.perf_counter() - t0, done


def host_threads() -> int:
    """Threads the oracle's matrix products run on (numpy's BLAS pool)."""
    try:
        import threadpoolctl

        info = threadpoolctl.threadpool_info()
        n = max((i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def host_info() -> dict:
    """The host the CPU legs ran on: logical CPUs available to this process and the CPU model."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except Exception:
        pass
    try:
        nproc = len(os.sched_getaffinity(0))
    except Exception:
        nproc = os.cpu_count()
    return {"nproc": nproc, "cpu_model": model, "blas_threads": host_threads()}


# The pages' own figures, quoted as context only (another machine, end-to-end or host-side; no kernel timing):
# techwalker article "华为巴黎研究院让AI视频“不再原地打转”", sections 二, 三 and 四.
PAGES_CONTEXT = {
    "end_to_end_generation_single_80GB_gpu": [
        {"model": "Wan 2.1 1.3B", "frames": 481, "dense_min": 51, "lvsa_min": 16, "speedup": 3.17},
        {"model": "Wan 2.1 14B", "frames": 481, "dense_min": 238, "lvsa_min": 80, "speedup": 2.98},
        {"model": "HunyuanVideo 1.5", "frames": 193, "dense_min": 80, "lvsa_min": 24, "speedup": 3.33},
    ],
    "host_window_extension": "about 1.4 us per frame, at most 200 us per step (section 二)",
    "host_anchor_recompute": "under 1 ms for the longest 121-frame sequence (section 三)",
    "source": "techwalker article, sections 二, 三, 四; context only, not a target",
}

# The list configurations of the five workloads (T, C, W), timed for the oracle's list build.
LIST_CONFIGS = {"tiny": (8, 4, 2), "wan1.3b_1x": (21, 21, 9), "wan1.3b_6x": (121, 21, 9), "wan14b_6x": (121, 21, 9),
                "hunyuan1.5_1.5x": (49, 33, 13)}


def oracle_list_build_us(steps: int = 50) -> dict:
    """The oracle's frame-list build (Python sets, by definition) timed per step over steps 0..steps-1 for
    the list configuration of every workload: median and max microseconds per step."""
    from oracle import lists as OL

    res = {}
    for name, (T, C, W) in LIST_CONFIGS.items():
        us = []
        for s in range(steps):
            t0 = time.perf_counter()
            OL.frame_lists(T, C, W, s)
            us.append((time.perf_counter() - t0) * 1e6)
        res[name] = {"T": T, "C": C, "W": W, "median_us": statistics.median(us), "max_us": max(us)}
    return res


def run_reference(args, rank, world):
    """The oracle as it stands, on the host cores: each step one bounded sample."""
    import synthetic

    if rank != 0:
        return 0
    w = synthetic.WORKLOADS[args.workload]
    per_step = args.ref_seconds or max(1.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_oracle_sample(w, per_step * 0.25)
    tot_f, tot_t, units = 0.0, 0.0, 0
    for _ in range(args.steps):
        f, t, u = cpu_oracle_sample(w, per_step)
        tot_f += f
        tot_t += t
        units += u
    value = tot_f / tot_t / 1e12
    ms_call = flops_per_call(w) / (value * 1e12) * 1e3
    sample = (f"{units} (head, query frame) units of {w.P} query rows each over {args.steps} steps "
              f"(~{per_step:.1f} s per step); value = sampled FLOPs / sampled time")
    info = host_info()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
        "full_call_ms_extrapolated": ms_call, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": info["blas_threads"], "kind": ORACLE_KIND,
                         "sample": sample, "nproc": info["nproc"], "cpu_model": info["cpu_model"]},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_cpu_full_calls(args, rank):
    """The oracle's whole call, timed on the host cores, for the two workloads small enough to finish in
    minutes: the tiny case (step 3) and Wan-1.3B at its 1x horizon (C = T: dense).  One JSON line."""
    import synthetic
    from oracle import attention as OA
    from oracle import lists as OL

    if rank != 0:
        return 0
    res = []
    for name, step in (("tiny", 3), ("wan1.3b_1x", 0)):
        w = synthetic.WORKLOADS[name]
        q, k, v = synthetic.make_qkv(w, device="cpu")
        t0 = time.perf_counter()
        lists = OL.frame_lists(w.T, w.C, w.W, step)
        OA.sparse_attention(q, k, v, lists, w.P)
        t = time.perf_counter() - t0
        res.append({"workload": name, "step": step, "seconds": t, "tflops": flops_per_call(w) / t / 1e12})
    info = host_info()
    print(json.dumps({"oracle_full_calls": res, "cores": info["blas_threads"], "nproc": info["nproc"],
                      "cpu_model": info["cpu_model"], "kind": ORACLE_KIND}), flush=True)
    return 0


def head_band(rank: int, world: int, H: int):
    """Heads [h0, h0 + n) of rank `rank` when H heads are split as evenly as possible over `world` ranks."""
    from block_sparse_attention_frame_b200.sequence_parallel import head_band as band

    return band(rank, world, H)


def workload_config(w, world, fixed_grid=False):
    return {"workload": w.name, "anchors": "fixed grid (step 0 pattern every step)" if fixed_grid else "rotating", "T": w.T, "tokens_per_frame": w.P, "heads": w.H, "head_dim": w.d, "C": w.C,
            "W": w.W, "G": max(0, w.C - w.W) if w.C < w.T else 0, "global_batch": w.B * world,
            "seq_len": w.T * w.P, "parallelism": "replicas" if world > 1 else "single",
            "l2": "inputs larger than L2 (Q+K+V+O working set "
                  f"{algorithmic_bytes(w) / 1e9:.2f} GB vs 126 MB), no flush"}


def run_lvsa(args, rank, world, local):
    import torch

    import block_sparse_attention_frame_b200 as lvsa
    import synthetic
    from block_sparse_attention_frame_b200.pipeline import StepPipeline, host_lists

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = synthetic.WORKLOADS[args.workload]
    q, k, v = synthetic.make_qkv(w, device=dev)
    w_full, h0, hn = w, 0, w.H
    shard = args.shard_heads and world > 1
    if shard:
        # one call split over the ranks by heads (heads are independent; the lists are shared): this rank
        # computes heads [h0, h0 + hn) of the same synthetic tensors, nothing is exchanged
        if world > w.H:
            raise SystemExit(f"--shard-heads needs at most {w.H} ranks")
        h0, hn = head_band(rank, world, w.H)
        q, k, v = (x[:, :, h0:h0 + hn].contiguous() for x in (q, k, v))
        w = synthetic.Workload(w.name, T=w.T, P=w.P, H=hn, d=w.d, C=w.C, W=w.W, B=w.B, seed=w.seed)
    F = flops_per_call(w)            # this rank's kernel
    F_call = flops_per_call(w_full)  # one whole call
    calls = 1 if shard else world    # per step, over all ranks: sharded ranks share one call
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)
    # the per-step path: host list build into a pinned ring buffer, async upload, kernel
    pipe = StepPipeline(w.T, w.C, w.W, w.P, dev, fixed_grid=args.fixed_grid)

    # ---------------------------------------------------------------- device-resident timing
    for s in range(args.warmup):
        pipe.step(s, q, k, v, out, stream)
    torch.cuda.synchronize()
    pipe.build_us.clear()
    ev_k = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        start.record(stream)
        for i in range(args.steps):
            pipe.step(args.warmup + i, q, k, v, out, stream, kernel_events=ev_k[i])
        stop.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = max_over_ranks(start.elapsed_time(stop), world)
    kernel_ms = [a.elapsed_time(b) for a, b in ev_k]
    build_us = list(pipe.build_us)
    status = lvsa.lvsa_get_device_status(clear=True)
    if status:
        raise RuntimeError(f"device status {status:#x} after the timed region")
    ms_per_step = elapsed_ms / args.steps
    value = calls * F_call * args.steps / (elapsed_ms * 1e-3) / 1e12
    if args.kernel_only:
        if rank == 0:
            print(json.dumps({"workload": w.name, "value": value, "unit": "TFLOP/s", "ms_per_step": ms_per_step,
                              "kernel_ms": kernel_ms, "clocks": clocks.summary()}), flush=True)
        return 0

    # ---------------------------------------------------------------- dense control (same kernel, C = T)
    # step by step: the sparse call of step s, then the same kernel with every frame listed
    dense_lists = torch.from_numpy(lvsa.lvsa_build_frame_lists(w.T, w.T, 1, 0)).to(dev)
    dout = torch.empty_like(q)
    lvsa.lvsa_attention(q, k, v, dense_lists, w.P, out=dout)
    torch.cuda.synchronize()
    ncmp = args.dense_compare_steps
    if ncmp < 0:
        ncmp = args.steps if w.name.startswith("hunyuan") else min(3, args.steps)
    per_step = []
    for i in range(ncmp):
        s = args.warmup + i
        es, ed = ((torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(2))
        pipe.step(s, q, k, v, out, stream, kernel_events=es)
        ed[0].record(stream)
        lvsa.lvsa_attention(q, k, v, dense_lists, w.P, out=dout, stream=stream)
        ed[1].record(stream)
        torch.cuda.synchronize()
        sp, dn = es[0].elapsed_time(es[1]), ed[0].elapsed_time(ed[1])
        per_step.append({"step": s, "sparse_ms": sp, "dense_ms": dn, "speedup": dn / sp})
    dense_ms = statistics.mean(x["dense_ms"] for x in per_step)
    del dout

    # ---------------------------------------------------------------- end to end with host buffers
    qh = q.cpu().pin_memory()
    kh = k.cpu().pin_memory()
    vh = v.cpu().pin_memory()
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    e2e_steps = max(3, min(args.steps, 10))
    # one pinned host list buffer per end-to-end step: the call copies it asynchronously
    e2e_lists = [torch.empty((w.T, w.L), dtype=torch.int32).pin_memory() for _ in range(e2e_steps + 1)]
    lists_dev = torch.empty((w.T, w.L), dtype=torch.int32, device=dev)

    def e2e_step(i, s):
        # the public host-buffer call: uploads of Q, K, V, the list and the readback of O are
        # inside it, pipelined against the kernel by bands of heads
        torch.cuda.nvtx.range_push("lvsa.build_lists")
        host_lists(w.T, w.C, w.W, s, args.fixed_grid, out=e2e_lists[i].numpy())
        torch.cuda.nvtx.range_pop()
        torch.cuda.nvtx.range_push("lvsa.attention_host")
        lvsa.lvsa_attention_host(qh, kh, vh, e2e_lists[i], w.P, oh, q, k, v, lists_dev, out,
                                 heads_per_band=args.heads_per_band, stream=stream)
        torch.cuda.nvtx.range_pop()

    e2e_step(e2e_steps, 0)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(e2e_steps):
        e2e_step(i, args.warmup + i)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    h2d = 3 * q.numel() * q.element_size() + w.T * w.L * 4
    d2h = out.numel() * out.element_size()

    # ---------------------------------------------------------------- roofline of the kernel
    peaks, peak_src = load_peaks()
    kern_avg_ms = sum(kernel_ms) / len(kernel_ms)
    achieved = F / (kern_avg_ms * 1e-3) / 1e12  # this rank's kernel (its heads when sharded)
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tpath) and not shard:
        try:
            with open(tpath) as f:
                tj = json.load(f)
            if tj.get("workload") == w.name and tj.get("kernel_source_hash") == kernel_source_hash():
                traffic = tj.get("bytes_per_launch")
        except Exception:
            traffic = None

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "strong" if shard else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": (dict(workload_config(w_full, 1, args.fixed_grid),
                        parallelism=f"heads split over {world} ranks (this rank {h0}..{h0 + hn - 1})")
                   if shard else workload_config(w, world, args.fixed_grid)),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{peak_src} bf16 dense (burst)",
                     "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained", peak)),
                     "kernel_ms_avg": kern_avg_ms, "flops_per_launch": F},
        "kernel_ms_over_steps": {"steps": f"s = {args.warmup}..{args.warmup + args.steps - 1}",
                                 "mean": kern_avg_ms, "median": statistics.median(kernel_ms),
                                 "min": min(kernel_ms), "max": max(kernel_ms)},
        "e2e": {"value": calls * F_call / (e2e_ms * 1e-3) / 1e12,
                "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "call": "lvsa_attention_host (pinned host buffers; copies pipelined by bands of "
                        f"{args.heads_per_band or 1} head(s))"},
        "gpu_launches": args.steps,
        "dense_control": {"ms_per_call": dense_ms, "tflops": flops_per_call_dense(w) / (dense_ms * 1e-3) / 1e12,
                          "speedup_sparse_vs_dense": statistics.mean(x["speedup"] for x in per_step),
                          "per_step": per_step},
        "list_build_us": {"median": statistics.median(build_us), "max": max(build_us),
                          "what": "lvsa_build_frame_lists (C ABI) into the pinned ring buffer, per timed step"},
        "clocks": clocks.summary(),
        "pages_context": PAGES_CONTEXT,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f, t, units = cpu_oracle_sample(w, args.cpu_seconds)
        info = host_info()
        line["cpu_baseline"] = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": info["blas_threads"],
                                "kind": ORACLE_KIND, "nproc": info["nproc"], "cpu_model": info["cpu_model"],
                                "sample": f"{units} (head, query frame) units of {w.P} rows, "
                                          f"{t:.1f} s of fp64 numpy on the host",
                                "list_build_us_per_step": oracle_list_build_us()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_sweep(args, rank, world, local):
    """Horizon sweep at the Wan-1.3B budget (C = 21, W = 9, H = 12, P = 1560): the same kernel with the
    LVSA lists and with dense lists (C = T) for T = 21 ... 257 latent frames; one JSON line per T."""
    import torch

    import block_sparse_attention_frame_b200 as lvsa
    import synthetic

    if rank != 0:
        return 0
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    base = synthetic.WORKLOADS["wan1.3b_6x"]
    for T in [int(x) for x in args.sweep_T.split(",")]:
        w = synthetic.Workload(f"wan1.3b_T{T}", T=T, P=base.P, H=base.H, d=base.d, C=base.C, W=base.W, seed=2000 + T)
        q, k, v = synthetic.make_qkv(w, device=dev)
        out = torch.empty_like(q)
        res = {}
        for kind, C in (("sparse", w.C), ("dense", T)):
            lists = torch.from_numpy(lvsa.lvsa_build_frame_lists(T, C, min(w.W, C), 7)).to(dev)
            calls = 3 if kind == "sparse" or T <= 121 else 1
            for _ in range(2):
                lvsa.lvsa_attention(q, k, v, lists, w.P, out=out)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(calls):
                lvsa.lvsa_attention(q, k, v, lists, w.P, out=out)
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / calls
            L = lists.shape[1]
            res[kind] = (ms, 4.0 * w.B * w.H * T * L * w.P * w.P * w.d / (ms * 1e-3) / 1e12)
        print(json.dumps({"sweep": "horizon", "T": T, "video_frames": 4 * (T - 1) + 1, "C": w.C, "W": w.W,
                          "sparse_ms": res["sparse"][0], "sparse_tflops": res["sparse"][1],
                          "dense_ms": res["dense"][0], "dense_tflops": res["dense"][1],
                          "speedup": res["dense"][0] / res["sparse"][0]}), flush=True)
        del q, k, v, out
        torch.cuda.empty_cache()
    return 0


def run_sequence_parallel(args, rank, world, local):
    """One call split over the ranks by token ranges (DeepSpeed-Ulysses layout, the pages' multi-device
    setting): rank r holds tokens of Q, K, V and of the output for every head; its band of heads is gathered
    from the other ranks by peer loads, and the attention stores each output row into its owner's buffer."""
    import torch

    import block_sparse_attention_frame_b200 as lvsa
    import synthetic
    from block_sparse_attention_frame_b200.sequence_parallel import SequenceParallelAttention

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = synthetic.WORKLOADS[args.workload]
    if world > w.H:
        raise SystemExit(f"--sequence-parallel needs at most {w.H} ranks")
    sp = SequenceParallelAttention(w.T, w.P, w.H, w.d, batch=w.B, device=dev)
    q, k, v = synthetic.make_qkv(w, device=dev)  # the same seeded tensors on every rank
    a, b = sp.starts[rank], sp.starts[rank + 1]
    for dst, src in ((sp.q, q), (sp.k, k), (sp.v, v)):
        dst.copy_(src[:, a:b])
    del q, k, v
    torch.cuda.empty_cache()
    stream = torch.cuda.current_stream(dev)
    nsteps = args.warmup + args.steps
    pinned = [torch.empty((w.T, w.L), dtype=torch.int32).pin_memory() for _ in range(nsteps)]
    lists_dev = torch.empty((w.T, w.L), dtype=torch.int32, device=dev)

    def step(s, events=None):
        lvsa.lvsa_build_frame_lists(w.T, w.C, w.W, s, out=pinned[s % nsteps].numpy())
        lists_dev.copy_(pinned[s % nsteps], non_blocking=True)
        sp(lists_dev, events=events)

    for s in range(args.warmup):
        step(s)
    torch.cuda.synchronize()
    events = []
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    with ClockSampler(local) as clocks:
        start.record(stream)
        for i in range(args.steps):
            step(args.warmup + i, events)
        stop.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = max_over_ranks(start.elapsed_time(stop), world)
    gather_ms = [e0.elapsed_time(e1) for e0, e1, _ in events]
    attn_ms = [e1.elapsed_time(e2) for _, e1, e2 in events]
    if lvsa.lvsa_get_device_status(clear=True):
        raise RuntimeError("device status set after the timed region")

    # end to end: this rank's token range of Q, K, V from pinned host memory, its output rows back, through
    # the host-buffer call of the sequence-parallel object (one rank: transfers pipelined by bands of heads)
    qh, kh, vh = (x.cpu().pin_memory() for x in (sp.q, sp.k, sp.v))
    oh = torch.empty(sp.out.shape, dtype=sp.out.dtype).pin_memory()
    e2e_steps = max(3, min(args.steps, 10))

    def e2e_step(s):
        lvsa.lvsa_build_frame_lists(w.T, w.C, w.W, s, out=pinned[s % nsteps].numpy())
        sp.host_call(qh, kh, vh, pinned[s % nsteps], oh)

    e2e_step(0)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps

    F_call = flops_per_call(w)
    F_band = 4.0 * w.B * sp.band * w.T * w.L * w.P * w.P * w.d
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    kern = sum(attn_ms) / len(attn_ms)
    achieved = F_band / (kern * 1e-3) / 1e12 if sp.band else 0.0
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if world == 1 and os.path.exists(tpath):
        with open(tpath) as f:
            tj = json.load(f)
        if tj.get("workload") == w.name and tj.get("kernel_source_hash") == kernel_source_hash():
            traffic = tj.get("bytes_per_launch")
    row_bytes = w.H * w.d * 2
    peer_bytes = 3 * w.B * (w.T * w.P - (b - a)) * sp.band * w.d * 2 if world > 1 else 0
    line = {
        "metric": METRIC, "value": F_call * args.steps / (elapsed_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(w, 1), parallelism=(
            f"sequence-parallel over {world} rank(s) (Ulysses layout): token ranges {sp.chunk_tokens}; "
            f"this rank heads {sp.head0}..{sp.head0 + sp.band - 1}; heads gathered by peer loads, output rows "
            "stored to their owners by the attention kernel")),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic, "peak_source": f"{peak_src} bf16 dense (burst)",
                     "kernel_ms_avg": kern, "flops_per_launch": F_band},
        "exchange": {"gather_ms_avg": sum(gather_ms) / len(gather_ms), "peer_bytes_read_per_step": peer_bytes,
                     "gather_GBps": (peer_bytes / (sum(gather_ms) / len(gather_ms) * 1e-3) / 1e9)
                     if peer_bytes else None},
        "e2e": {"value": F_call / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": 3 * w.B * (b - a) * row_bytes + w.T * w.L * 4,
                "d2h_bytes_per_step": w.B * (b - a) * row_bytes,
                "call": "SequenceParallelAttention.host_call on this rank's token range (pinned host buffers; "
                        "one rank: lvsa_attention_host, transfers pipelined by bands of heads)"},
        "gpu_launches": args.steps * (2 if world > 1 else 1),
        "clocks": clocks.summary(),
    }
    if world == 1 and w.B == 1:
        line["exchange"]["gather_local"] = gather_local_roofline(w, sp, peaks, peak_src)
    sp.close()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def gather_local_roofline(w, sp, peaks, peak_src, ranks=8, calls=10):
    """The band gather of rank 0 of an emulated `ranks`-way split, on this GPU: the source ranges are token
    ranges of the resident Q, K, V (contiguous for batch 1), the band buffers are local.  An HBM-bound copy:
    bytes = read + write of 3 tensors x tokens x band x d x 2."""
    import torch

    import block_sparse_attention_frame_b200 as lvsa
    from block_sparse_attention_frame_b200.sequence_parallel import head_band, token_ranges

    tokens = w.T * w.P
    n = token_ranges(tokens, ranks)
    starts = [sum(n[:r]) for r in range(ranks)]
    row = w.H * w.d * 2
    tables = [[x.data_ptr() + s0 * row for s0 in starts] for x in (sp.q, sp.k, sp.v)]
    h0, band = head_band(0, ranks, w.H)
    bufs = [torch.empty((1, tokens, band, w.d), dtype=torch.bfloat16, device=sp.q.device) for _ in range(3)]
    for _ in range(3):
        lvsa.lvsa_seq_to_heads(*tables, n, h0, band, *bufs, heads=w.H)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(calls):
        lvsa.lvsa_seq_to_heads(*tables, n, h0, band, *bufs, heads=w.H)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / calls
    ok = all(torch.equal(b.view(torch.int16), x[:, :, h0:h0 + band].view(torch.int16))
             for b, x in zip(bufs, (sp.q, sp.k, sp.v)))
    nbytes = 2 * 3 * tokens * band * w.d * 2
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    return {"ranks_emulated": ranks, "band_heads": band, "ms": ms, "bytes": nbytes,
            "GBps": nbytes / (ms * 1e-3) / 1e9, "frac_of_hbm": nbytes / (ms * 1e-3) / 1e9 / hbm,
            "hbm_peak_source": f"{peak_src} copy bandwidth", "equal_to_source_heads": ok}


def flops_per_call_dense(w) -> float:
    return 4.0 * w.B * w.H * w.T * w.T * w.P * w.P * w.d


def kernel_source_hash() -> str:
    import hashlib

    h = hashlib.sha256()
    # the device code only: host-side changes (launch plumbing, entry points) leave the counters valid
    for rel in ("block_sparse_attention_frame_b200/csrc/attention_kernel.cuh",
                "block_sparse_attention_frame_b200/csrc/sm100.cuh"):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="lvsa", choices=["lvsa", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fixed-grid", action="store_true",
                    help="ablation: anchors do not rotate (the step-0 pattern at every step)")
    ap.add_argument("--sweep", choices=["horizon"], default=None,
                    help="horizon sweep: sparse vs dense for several T (one JSON line per T)")
    ap.add_argument("--sweep-T", default="21,41,81,121,161,257")
    ap.add_argument("--kernel-only", action="store_true",
                    help="time the device path only and print a short line (for profiling runs)")
    ap.add_argument("--ref-seconds", type=float, default=0.0, help="reference arm: CPU seconds per step")
    ap.add_argument("--shard-heads", action="store_true",
                    help="with --gpus N > 1: split one call over the ranks by heads (strong scaling) "
                         "instead of running a replica per rank")
    ap.add_argument("--sequence-parallel", action="store_true",
                    help="split one call over the ranks by token ranges (Ulysses layout, peer-memory exchanges)")
    ap.add_argument("--dense-compare-steps", type=int, default=-1,
                    help="steps timed sparse then dense (C = T) one after the other (-1: every timed step for "
                         "the HunyuanVideo workloads, 3 otherwise)")
    ap.add_argument("--cpu-full-calls", action="store_true",
                    help="time the oracle's full call on the tiny and Wan-1.3B 1x workloads (minutes of CPU) "
                         "and print one JSON line")
    ap.add_argument("--heads-per-band", type=int, default=0,
                    help="end-to-end call: heads per pipelined band (0: one)")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps; the JSON reports the count used
    rank, world, local = dist_setup(args)
    try:
        if args.impl == "reference":
            return run_reference(args, rank, world)
        if args.cpu_full_calls:
            return run_cpu_full_calls(args, rank)
        if args.sweep:
            return run_sweep(args, rank, world, local)
        if args.sequence_parallel:
            return run_sequence_parallel(args, rank, world, local)
        return run_lvsa(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
