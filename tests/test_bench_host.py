"""Host-side logic of bench.py (no GPU): FLOP model, clock parsing, the
reference arm's JSON line, and max-over-ranks timing with 2 gloo ranks."""

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_flop_model_matches_workload_figures():
    from synthetic import WORKLOADS

    assert bench.flops_per_call(WORKLOADS["wan1.3b_6x"]) / 1e12 == pytest.approx(37.993, rel=1e-4)
    assert bench.flops_per_call(WORKLOADS["wan14b_6x"]) / 1e12 == pytest.approx(126.64, rel=1e-4)
    assert bench.flops_per_call(WORKLOADS["hunyuan1.5_1.5x"]) / 1e12 == pytest.approx(32.24, rel=1e-3)
    assert bench.flops_per_call_dense(WORKLOADS["wan1.3b_6x"]) / 1e12 == pytest.approx(218.9, rel=1e-3)
    assert bench.algorithmic_bytes(WORKLOADS["wan1.3b_6x"]) / 1e9 == pytest.approx(2.32, rel=1e-2)


def test_clock_summary_parsing():
    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.lines = [
        "1965, 1965, 120.5, 0x0, Not Active, Not Active, Not Active, Not Active",
        "1500, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "1400, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active",
        "garbage line",
    ]
    s = cs.summary()
    assert s["sm_mhz"] == 1450 and s["sm_max_mhz"] == 1965 and s["reasons"] == ["sw_power_cap"]
    assert s["samples"] == 3 and s["samples_under_load"] == 2


def test_reference_arm_json_line(capsys):
    rc = bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3",
                     "--ref-seconds", "0.05"])
    assert rc == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    cb = line["cpu_baseline"]
    assert cb["kind"].startswith("oracle") and cb["value"] == line["value"]
    assert cb["cores"] >= 1 and cb["nproc"] >= 1 and "cpu_model" in cb
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["config"]["workload"] == "tiny"
    # ms_per_step is what one step of the arm took (a bounded sample); the full call is extrapolated apart
    assert 0 < line["ms_per_step"] < 5000
    assert line["full_call_ms_extrapolated"] > 0


def test_reference_arm_does_not_load_the_cuda_library():
    """The oracle arm imports the input generator and the oracle only: the CUDA library stays unloaded."""
    code = (
        "import sys, json; sys.path.insert(0, %r); import bench; "
        "rc = bench.main(['--impl', 'reference', '--workload', 'tiny', '--steps', '1', '--warmup', '3', "
        "'--ref-seconds', '0.02']); "
        "maps = open('/proc/self/maps').read(); "
        "print('LOADED' if 'liblvsa' in maps else 'NOT_LOADED'); "
        "print('PKG' if 'block_sparse_attention_frame_b200' in sys.modules else 'NO_PKG')" % ROOT)
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300,
                         env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
    assert res.returncode == 0, res.stderr[-2000:]
    assert "NOT_LOADED" in res.stdout and "NO_PKG" in res.stdout, res.stdout


def test_oracle_list_build_timing_and_page_context():
    t = bench.oracle_list_build_us(steps=3)
    assert set(t) == set(bench.LIST_CONFIGS)
    for name, r in t.items():
        assert (r["T"], r["C"], r["W"]) == bench.LIST_CONFIGS[name]
        assert 0 < r["median_us"] <= r["max_us"]
    ctx = bench.PAGES_CONTEXT["end_to_end_generation_single_80GB_gpu"][0]
    assert (ctx["dense_min"], ctx["lvsa_min"], ctx["speedup"]) == (51, 16, 3.17)
    info = bench.host_info()
    assert info["nproc"] >= 1 and info["blas_threads"] >= 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


WORKER = r"""
import os, sys
sys.path.insert(0, {root!r})
import torch.distributed as dist
import bench
rank = int(os.environ["RANK"])
dist.init_process_group("gloo")
v = bench.max_over_ranks(10.0 + rank * 5.0, 2)
bench.barrier(2)
print("RESULT", rank, v, flush=True)
dist.destroy_process_group()
"""


def test_max_over_ranks_two_gloo_ranks(tmp_path):
    port = _free_port()
    script = tmp_path / "worker.py"
    script.write_text(WORKER.format(root=ROOT))
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                   CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.STDOUT, text=True))
    outs = [p.communicate(timeout=120)[0] for p in procs]
    for rank, (p, out) in enumerate(zip(procs, outs)):
        assert p.returncode == 0, out
        assert f"RESULT {rank} 15.0" in out, out


def test_reference_arm_nonzero_rank_exits_without_work():
    class A:
        workload = "tiny"
        steps = 1
        warmup = 3
        ref_seconds = 0.01

    assert bench.run_reference(A, rank=1, world=2) == 0


def test_head_bands_cover_every_head_once():
    for H in range(1, 41):
        for world in range(1, min(H, 8) + 1):
            bands = [bench.head_band(r, world, H) for r in range(world)]
            covered = [h for h0, n in bands for h in range(h0, h0 + n)]
            assert covered == list(range(H))
            sizes = [n for _, n in bands]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
