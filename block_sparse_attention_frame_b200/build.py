"""Build step of the in-tree C-ABI library ``liblvsa.so`` (sm_100a).

``python block_sparse_attention_frame_b200/build.py [--force] [--ptxas-v]``
compiles ``csrc/*.cpp`` and ``csrc/*.cu`` with nvcc for sm_100a into
``block_sparse_attention_frame_b200/liblvsa.so``.  nvcc cross-compiles, so this
runs on a machine without a GPU.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(PKG, "liblvsa.so")

SOURCES = ["lists.cpp", "attention.cu", "exchange.cu"]
HEADERS = [os.path.join(INCLUDE, "lvsa.h"), os.path.join(CSRC, "sm100.cuh"), os.path.join(CSRC, "attention_kernel.cuh"),
           os.path.join(CSRC, "buffer_checks.h")]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build liblvsa.so")


def _inputs():
    return [os.path.join(CSRC, s) for s in SOURCES] + HEADERS + [os.path.abspath(__file__)]


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def build_library(force: bool = False, quiet: bool = False, ptxas_verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB_PATH
    cmd = [
        nvcc_path(),
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-lineinfo", "-std=c++17",
        "-Xcompiler", "-fPIC", "-shared",
        "-I", INCLUDE, "-I", CSRC,
        *[os.path.join(CSRC, s) for s in SOURCES],
        "-o", LIB_PATH + ".tmp",
    ]
    if ptxas_verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    os.replace(LIB_PATH + ".tmp", LIB_PATH)
    if not quiet or ptxas_verbose:
        sys.stdout.write(res.stdout + res.stderr)
    return LIB_PATH


if __name__ == "__main__":
    build_library(force="--force" in sys.argv, ptxas_verbose="--ptxas-v" in sys.argv)
    print(LIB_PATH)
