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
    assert call(lists=A + 4 * M + 256) == INV  # the output overlaps the device lists
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
    assert call(lists_dev=A + 12 * n + 64) == INV  # output staging overlaps the device lists
    assert call(lists_host=A + 4 * n + 64) == INV  # host output overlaps the host lists
    assert call(L=0) == INV and call(T=0) == INV
    assert call(d=96) == lib.LVSA_ERR_UNSUPPORTED
    from conftest import cuda_available

    if not cuda_available():
        assert call() in (lib.LVSA_ERR_CUDA, lib.LVSA_ERR_UNSUPPORTED)


def test_seq_to_heads_argument_validation_without_gpu(lib):
    A, M = 1 << 24, 1 << 20  # fake 16-byte aligned addresses 1 MB apart
    good = dict(q=[A, A + M], k=[A + 2 * M, A + 3 * M], v=[A + 4 * M, A + 5 * M], n=[64, 64], H=4, h0=1, band=2,
                d=64, B=1, qb=A + 8 * M, kb=A + 9 * M, vb=A + 10 * M)

    def call(**kw):
        a = dict(good, **kw)
        return lib.lvsa_seq_to_heads_raw(a["q"], a["k"], a["v"], a["n"], a["H"], a["h0"], a["band"], a["d"], a["B"],
                                         a["qb"], a["kb"], a["vb"])

    INV = lib.LVSA_ERR_INVALID_ARG
    assert call(q=[0, A + M]) == INV              # a range with tokens needs a buffer
    assert call(q=[0, A + M], n=[0, 128]) != INV  # ... an empty one does not
    assert call(q=[A + 8, A + M]) == INV          # misaligned source
    assert call(qb=A + 8 * M + 8) == INV          # misaligned destination
    assert call(n=[-1, 64]) == INV
    assert call(n=[0, 0]) == INV                  # no token at all
    assert call(h0=3) == INV                      # band past the last head
    assert call(band=0) == INV
    assert call(h0=-1) == INV
    assert call(B=0) == INV
    assert call(kb=A + 8 * M) == INV              # two band buffers overlap
    assert call(qb=A + M) == INV                  # a band buffer overlaps a local range buffer
    assert call(d=96) == lib.LVSA_ERR_UNSUPPORTED
    assert lib.lvsa_seq_to_heads_raw([A] * 65, [A] * 65, [A] * 65, [1] * 65, 4, 0, 1, 64, 1, A + 8 * M, A + 9 * M,
                                     A + 10 * M) == INV  # more ranges than a launch takes
    assert call() in (lib.LVSA_ERR_CUDA, lib.LVSA_ERR_UNSUPPORTED)  # valid: fails only at the CUDA step


def test_attention_to_chunks_argument_validation_without_gpu(lib):
    A, M = 1 << 24, 1 << 20
    T, P, H, d = 8, 64, 2, 64
    good = dict(q=A, k=A + M, v=A + 2 * M, lists=A + 3 * M, L=4, T=T, P=P, H=H, d=d, B=1, scale=0.0,
                outs=[A + 4 * M, A + 5 * M, A + 6 * M], n=[100, 0, T * P - 100], out_heads=4, h0=2)

    def call(**kw):
        a = dict(good, **kw)
        return lib.lvsa_attention_to_chunks_raw(a["q"], a["k"], a["v"], a["lists"], a["L"], a["T"], a["P"], a["H"],
                                                a["d"], a["B"], a["scale"], a["outs"], a["n"], a["out_heads"],
                                                a["h0"])

    INV = lib.LVSA_ERR_INVALID_ARG
    assert call(n=[100, 0, T * P - 101]) == INV     # ranges must cover the sequence exactly
    assert call(n=[100, 0, T * P]) == INV
    assert call(n=[100, -1, T * P - 99]) == INV
    assert call(outs=[0, A + 5 * M, A + 6 * M]) == INV  # a non-empty range needs a buffer
    assert call(outs=[A + 4 * M, 0, A + 6 * M]) != INV  # an empty range does not
    assert call(outs=[A + 4 * M + 8, A + 5 * M, A + 6 * M]) == INV
    assert call(outs=[A + 4 * M, A + 5 * M, A + 2 * M]) == INV  # an output buffer overlaps v
    assert call(outs=[A + 4 * M, A + 5 * M, A + 4 * M + 256]) == INV  # two output buffers overlap
    assert call(outs=[A + 4 * M, A + 5 * M, A + 3 * M]) == INV  # an output buffer overlaps the lists
    assert call(outs=[A + 4 * M, A + 4 * M, A + 6 * M]) != INV  # an empty range may share an address
    assert call(h0=3) == INV                        # heads past out_heads
    assert call(out_heads=1) == INV
    assert call(h0=-1) == INV
    assert call(outs=[A + 4 * M] * 65, n=[T * P] + [0] * 64) == INV  # more ranges than a launch takes
    assert call(q=0) == INV
    assert call(L=9) == INV
    assert call(d=96) == lib.LVSA_ERR_UNSUPPORTED
    assert call() in (lib.LVSA_ERR_CUDA, lib.LVSA_ERR_UNSUPPORTED)


def test_ipc_calls_reject_null_and_unknown_pointers(lib):
    import ctypes

    assert lib._lib.lvsa_ipc_export(None, ctypes.create_string_buffer(lib.LVSA_IPC_HANDLE_BYTES)) == \
        lib.LVSA_ERR_INVALID_ARG
    assert lib._lib.lvsa_ipc_import(None, ctypes.byref(ctypes.c_void_p())) == lib.LVSA_ERR_INVALID_ARG
    assert lib._lib.lvsa_ipc_release(None) == lib.LVSA_ERR_INVALID_ARG
    assert lib._lib.lvsa_ipc_release(ctypes.c_void_p(1 << 24)) == lib.LVSA_ERR_INVALID_ARG  # never imported
    with pytest.raises(ValueError):
        lib.lvsa_ipc_import(b"short")


def test_attention_joint_argument_validation_without_gpu(lib):
    A, M = 1 << 24, 1 << 20
    good = dict(q=A, k=A + M, v=A + 2 * M, lists=A + 3 * M, L=4, T=8, P=64, text=32, H=2, d=64, B=1, scale=0.0,
                out=A + 4 * M)

    def call(**kw):
        a = dict(good, **kw)
        return lib.lvsa_attention_joint_raw(a["q"], a["k"], a["v"], a["lists"], a["L"], a["T"], a["P"], a["text"],
                                            a["H"], a["d"], a["B"], a["scale"], a["out"], 0)

    INV = lib.LVSA_ERR_INVALID_ARG
    assert call(text=-1) == INV
    assert call(T=1, L=1, P=1 << 30, text=1 << 30) == INV  # video tokens fit, video + text pass INT_MAX
    assert call(out=A + 2 * M + 16) == INV               # output overlaps v
    assert call(lists=A + 4 * M + 32) == INV             # output overlaps the lists
    assert call(q=0) == INV
    assert call(L=9) == INV
    assert call(d=96) == lib.LVSA_ERR_UNSUPPORTED
    assert call() in (lib.LVSA_ERR_CUDA, lib.LVSA_ERR_UNSUPPORTED)
    assert call(text=0) in (lib.LVSA_ERR_CUDA, lib.LVSA_ERR_UNSUPPORTED)


def test_host_static_argument_validation_without_gpu(lib):
    """The allocation-free call validates everything, the size limit included, before any CUDA call."""
    A = 1 << 24
    M = 1 << 20
    good = dict(q=A, k=A + M, v=A + 2 * M, lists=A + 3 * M, L=4, T=8, P=64, H=2, d=64, B=1, scale=0.0,
                out=A + 4 * M)

    def call(**kw):
        a = dict(good, **kw)
        return lib.lvsa_attention_host_static_raw(a["q"], a["k"], a["v"], a["lists"], a["L"], a["T"], a["P"],
                                                  a["H"], a["d"], a["B"], a["scale"], a["out"], 0)

    INV = lib.LVSA_ERR_INVALID_ARG
    for name in ("q", "k", "v", "lists", "out"):
        assert call(**{name: 0}) == INV, name
    assert call(L=0) == INV
    assert call(L=9) == INV
    assert call(T=0) == INV
    assert call(P=0) == INV
    assert call(H=0) == INV
    assert call(B=0) == INV
    assert call(scale=float("nan")) == INV
    assert call(d=96) == lib.LVSA_ERR_UNSUPPORTED
    assert call(out=A + 64) == INV       # output overlaps q (each tensor is 128 KB here)
    assert call(lists=A + 4 * M + 64) == INV   # lists inside the output
    # Q, K, V and the output (each rounded up to 256 bytes) plus the lists must fit in the static array
    n = lib.LVSA_STATIC_SCRATCH_BYTES
    big = dict(q=A, k=A + n, v=A + 2 * n, lists=A + 3 * n, out=A + 4 * n, d=128, H=1, L=7)
    assert call(T=32, P=2048, **big) == INV           # 4 x 16 MiB: nothing left for the lists
    assert call(**dict(big, L=1), T=1, P=1 << 20) == INV   # one tensor alone beyond a quarter of the array
    from conftest import cuda_available

    if not cuda_available():
        # the largest of these shapes that fits passes validation and stops at the device check
        assert call(T=31, P=2048, **big) in (lib.LVSA_ERR_CUDA, lib.LVSA_ERR_UNSUPPORTED)
