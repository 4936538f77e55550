"""The library's host-side buffer decisions (csrc/buffer_checks.h), driven from a small C++ program with
fabricated CUDA pointer attributes and a stand-in for the peer-access calls (no GPU, no CUDA runtime):

* own device memory: usable as is;
* another GPU's memory: only where peer access is possible, and peer access is enabled (enabling it twice is
  not an error); a failed query or a failed enable refuses the buffer;
* pinned host and managed memory: usable, released at system scope; pageable memory: refused;
* byte-range overlap and the wait-budget conversion (ns -> cycles at 2 GHz) with its upper bound.
"""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = "/usr/local/cuda/include"

INV, CUDA_ERR = 1, 3


@pytest.mark.skipif(shutil.which("g++") is None or not os.path.isdir(CUDA_INC), reason="needs g++ and CUDA headers")
def test_buffer_decisions(tmp_path):
    exe = tmp_path / "buffer_checks_test"
    subprocess.run(["g++", "-std=c++17", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(ROOT, "block_sparse_attention_frame_b200", "csrc"), "-I", CUDA_INC,
                    os.path.join(ROOT, "tests", "buffer_checks_test.cpp"), "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True, timeout=60).stdout.splitlines()
    rows = {}
    for line in out:
        name, rest = line.split(" ", 1)
        rows[name] = rest
    P = "0x7f0000001000"
    assert rows["own"] == f"status=0 ptr={P} remote=0 enable=0 clear=0"
    assert rows["peer"] == f"status=0 ptr={P} remote=1 enable=1 clear=0"
    assert rows["peer_enabled"] == f"status=0 ptr={P} remote=1 enable=1 clear=1"
    assert rows["peer_enable_fails"].startswith(f"status={CUDA_ERR} ")
    assert rows["peer_no_access"].startswith(f"status={INV} ") and rows["peer_no_access"].endswith("enable=0 clear=0")
    assert rows["peer_query_fails"].startswith(f"status={INV} ")
    assert rows["pinned_host"] == f"status=0 ptr={P} remote=1 enable=0 clear=0"
    assert rows["managed"] == f"status=0 ptr={P} remote=1 enable=0 clear=0"
    assert rows["pageable"].startswith(f"status={INV} ")
    assert rows["no_device_ptr"].startswith(f"status={INV} ")
    assert rows["disjoint"] == "1 0 0 1 0"
    assert rows["cycles"] == "2000 8000000000 2000000000000"


def test_wait_budget_bounds(lib):
    assert lib._lib.lvsa_set_wait_budget_ns(10 ** 12) == 0
    assert lib._lib.lvsa_set_wait_budget_ns(10 ** 12 + 1) == lib.LVSA_ERR_INVALID_ARG
    assert lib._lib.lvsa_set_wait_budget_ns(2 ** 64 - 1) == lib.LVSA_ERR_INVALID_ARG
    assert lib._lib.lvsa_set_wait_budget_ns(0) == 0  # raised to the 1000 ns minimum
    assert lib._lib.lvsa_set_wait_budget_ns(4_000_000_000) == 0  # back to the default
