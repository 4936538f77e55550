"""The C ABI from plain C: a small C program (tests/c_abi_consumer.c) is compiled with gcc against
include/lvsa.h, linked to liblvsa.so and run; its frame lists must equal the hand-derived golden table and
its refused calls must report the documented status codes.  No GPU needed."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_uses_the_abi(lib, tmp_path):
    exe = tmp_path / "c_abi_consumer"
    pkg = os.path.dirname(lib.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_consumer.c"), "-L", pkg, "-llvsa",
                    f"-Wl,-rpath,{pkg}", "-o", str(exe)], check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True, timeout=120).stdout.splitlines()
    golden = [l.strip() for l in open(os.path.join(ROOT, "tests", "golden", "worked_example_T8_C4_W2.txt"))
              if l.strip() and not l.startswith("#")]
    assert out[:24] == golden
    assert out[24] == "anchors LVSA_OK G=2 1 5"
    assert out[25] == "null q: LVSA_ERR_INVALID_ARG"
    assert out[26] == "d=96: LVSA_ERR_UNSUPPORTED"
    assert out[27] == "small buffer: LVSA_ERR_BUFFER_TOO_SMALL"
    assert out[28].startswith("version ")
