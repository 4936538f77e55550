"""The C-ABI library loads and exports every symbol include/lvsa.h declares;
argument validation happens before any CUDA call (no GPU needed)."""

import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "lvsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lvsa_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("lvsa_build_frame_lists", "lvsa_attention", "lvsa_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lib.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib._lib, name)
    assert set(lib.EXPORTED) == set(declared_functions())


def test_status_strings(lib):
    assert lib.status_string(0) == "LVSA_OK"
    assert lib.status_string(4) == "LVSA_ERR_TIMEOUT"
    assert lib.status_string(99) == "LVSA_ERR_UNKNOWN"
    assert lib.lvsa_version() >= 100


def test_attention_argument_validation_without_gpu(lib):
    A = 1 << 24  # 16-byte aligned fake addresses 1 MB apart (no overlap); validation fails before any is used
    M = 1 << 20
    good = dict(q=A, k=A + M, v=A + 2 * M, lists=A + 3 * M, L=4, T=8, P=64, H=2, d=64, B=1, scale=0.0,
                out=A + 4 * M, stream=0)

    def call(**kw):
        a = dict(good, **kw)
        return lib.lvsa_attention_raw(a["q"], a["k"], a["v"], a["lists"], a["L"], a["T"], a["P"], a["H"],
                                      a["d"], a["B"], a["scale"], a["out"], a["stream"])

    INV = lib.LVSA_ERR_INVALID_ARG
    assert call(q=0) == INV
    assert call(lists=0) == INV
    assert call(out=0) == INV
    assert call(L=0) == INV
    assert call(L=9) == INV
    assert call(T=0) == INV
    assert call(P=0) == INV
    assert call(H=0) == INV
    assert call(B=0) == INV
    assert call(out=A) == INV            # aliases q
    assert call(out=A + 64) == INV       # overlaps q (and k, v) without being equal
    assert call(q=A + 8) == INV          # not 16-byte aligned
    assert call(lists=A + 3 * M + 2) == INV  # int32 misaligned
    assert call(scale=float("nan")) == INV
    assert call(T=1 << 20, P=1 << 12) == INV  # T*P overflows int32
    assert call(d=96) == lib.LVSA_ERR_UNSUPPORTED
    assert call(T=4097, L=4) == lib.LVSA_ERR_UNSUPPORTED   # frame bitmaps cover up to 4096 latent frames
    # valid arguments on a machine without a B200: a clean error, never a crash
    from conftest import cuda_available

    if not cuda_available():
        assert call() in (lib.LVSA_ERR_CUDA, lib.LVSA_ERR_UNSUPPORTED)


def test_host_path_argument_validation_without_gpu(lib):
    A = 1 << 20       # 16-byte aligned fake addresses; validation fails before any is used
    n = 8 * 64 * 2 * 64 * 2   # bytes of one [1, 8*64, 2, 64] bf16 tensor
    good = [A, A + n, A + 2 * n, A + 3 * n, 4, 8, 64, 2, 64, 1, 0.0, A + 4 * n,
            A + 8 * n, A + 9 * n, A + 10 * n, A + 11 * n, A + 12 * n, 0, 0]
    names = ["q_host", "k_host", "v_host", "lists_host", "L", "T", "P", "H", "d", "B", "scale", "out_host",
             "q_dev", "k_dev", "v_dev", "lists_dev", "out_dev", "heads_per_band", "stream"]

    def call(**kw):
        a = list(good)
        for key, val in kw.items():
            a[names.index(key)] = val
        return lib.lvsa_attention_host_raw(*a)

    INV = lib.LVSA_ERR_INVALID_ARG
    for ptr in ("q_host", "k_host", "v_host", "lists_host", "out_host", "q_dev", "k_dev", "v_dev", "lists_dev",
                "out_dev"):
        assert call(**{ptr: 0}) == INV, ptr
    assert call(heads_per_band=-1) == INV
    assert call(heads_per_band=3) == INV          # more than the 2 heads
    assert call(q_dev=A + 8 * n + 8) == INV       # device staging not 16-byte aligned
    assert call(lists_dev=A + 11 * n + 2) == INV  # int32 misaligned
    assert call(out_dev=A + 8 * n + 64) == INV    # output staging overlaps q_dev
    assert call(out_host=A + n // 2) == INV       # host output overlaps q_host
    assert call(L=0) == INV and call(T=0) == INV
    assert call(d=96) == lib.LVSA_ERR_UNSUPPORTED
    from conftest import cuda_available

    if not cuda_available():
        assert call() in (lib.LVSA_ERR_CUDA, lib.LVSA_ERR_UNSUPPORTED)
