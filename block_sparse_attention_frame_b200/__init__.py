"""Python binding of the LVSA B200 library (``liblvsa.so``).

Argument marshalling only: every step of the path runs in the C++/CUDA
library.  PyTorch supplies device memory and streams.  If the library is not
built this module raises on import; there is no CPU or PyTorch fallback.

Functions carry the C ABI's names (declared in ``include/lvsa.h``):

``lvsa_build_frame_lists(T, C, W, step)`` -> int32 numpy array [T, min(C,T)]
``lvsa_build_anchors(T, C, W, step)``     -> int32 numpy array [G]
``lvsa_attention(q, k, v, lists, tokens_per_frame, scale=0, out=None, stream=None)``
``lvsa_attention_joint(q, k, v, lists, tokens_per_frame, scale=0, out=None, stream=None)`` (video + text)
``lvsa_attention_host(q_host, k_host, v_host, lists_host, tokens_per_frame, out_host, q_dev, k_dev, v_dev,
lists_dev, out_dev, scale=0, heads_per_band=0, stream=None)``
``lvsa_attention_host_static(q_host, k_host, v_host, lists_host, tokens_per_frame, out_host, scale=0, stream=None)``
(no allocation, no caller device buffer)
``lvsa_seq_to_heads(q_chunks, k_chunks, v_chunks, chunk_tokens, head0, band, q_band, k_band, v_band, stream=None)``
``lvsa_attention_to_chunks(q, k, v, lists, tokens_per_frame, out_chunks, chunk_tokens, out_heads, head0, scale=0,
stream=None)``
``lvsa_ipc_export(tensor)`` -> bytes, ``lvsa_ipc_import(handle)`` -> int, ``lvsa_ipc_release(ptr)``
``lvsa_get_device_status(clear=False)``   -> int (LVSA_DEV_* bits)
``lvsa_set_wait_budget_ns(ns)``, ``lvsa_watchdog_selftest(budget_ns, stream=None)``
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblvsa.so")

LVSA_OK = 0
LVSA_ERR_INVALID_ARG = 1
LVSA_ERR_UNSUPPORTED = 2
LVSA_ERR_CUDA = 3
LVSA_ERR_TIMEOUT = 4
LVSA_ERR_BUFFER_TOO_SMALL = 5
LVSA_ERR_BAD_LIST = 6
LVSA_DEV_TIMEOUT = 0x1
LVSA_DEV_BAD_LIST = 0x2
LVSA_IPC_HANDLE_BYTES = 72
LVSA_STATIC_SCRATCH_BYTES = 64 << 20

EXPORTED = [
    "lvsa_build_frame_lists", "lvsa_build_anchors", "lvsa_attention", "lvsa_attention_host", "lvsa_get_device_status",
    "lvsa_set_wait_budget_ns", "lvsa_watchdog_selftest", "lvsa_status_string",
    "lvsa_version", "lvsa_seq_to_heads", "lvsa_attention_to_chunks", "lvsa_ipc_export", "lvsa_ipc_import",
    "lvsa_ipc_release", "lvsa_attention_joint", "lvsa_attention_host_static",
]


class LvsaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")


if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python block_sparse_attention_frame_b200/build.py` "
        "(there is no fallback path)")

_lib = ctypes.CDLL(LIB_PATH)
_c_int, _c_size, _c_ll, _c_ull, _c_float, _c_vp = (ctypes.c_int, ctypes.c_size_t, ctypes.c_longlong,
                                                     ctypes.c_ulonglong, ctypes.c_float, ctypes.c_void_p)
_i32p = ctypes.POINTER(ctypes.c_int32)

_lib.lvsa_build_frame_lists.argtypes = [_c_int, _c_int, _c_int, _c_ll, _i32p, _c_size, ctypes.POINTER(_c_int)]
_lib.lvsa_build_frame_lists.restype = _c_int
_lib.lvsa_build_anchors.argtypes = [_c_int, _c_int, _c_int, _c_ll, _i32p, _c_size, ctypes.POINTER(_c_int)]
_lib.lvsa_build_anchors.restype = _c_int
_lib.lvsa_attention.argtypes = [_c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                _c_float, _c_vp, _c_vp]
_lib.lvsa_attention.restype = _c_int
_lib.lvsa_attention_joint.argtypes = [_c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                      _c_int, _c_float, _c_vp, _c_vp]
_lib.lvsa_attention_joint.restype = _c_int
_lib.lvsa_attention_host.argtypes = [_c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                     _c_float, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_vp]
_lib.lvsa_attention_host.restype = _c_int
_lib.lvsa_attention_host_static.argtypes = [_c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_int, _c_int, _c_int, _c_int,
                                            _c_int, _c_float, _c_vp, _c_vp]
_lib.lvsa_attention_host_static.restype = _c_int
_lib.lvsa_seq_to_heads.argtypes = [_c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                   _c_vp, _c_vp, _c_vp, _c_vp]
_lib.lvsa_seq_to_heads.restype = _c_int
_lib.lvsa_attention_to_chunks.argtypes = [_c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                          _c_float, _c_vp, _c_vp, _c_int, _c_int, _c_int, _c_vp]
_lib.lvsa_attention_to_chunks.restype = _c_int
_lib.lvsa_ipc_export.argtypes = [_c_vp, _c_vp]
_lib.lvsa_ipc_export.restype = _c_int
_lib.lvsa_ipc_import.argtypes = [_c_vp, ctypes.POINTER(_c_vp)]
_lib.lvsa_ipc_import.restype = _c_int
_lib.lvsa_ipc_release.argtypes = [_c_vp]
_lib.lvsa_ipc_release.restype = _c_int
_lib.lvsa_get_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint), _c_int]
_lib.lvsa_get_device_status.restype = _c_int
_lib.lvsa_set_wait_budget_ns.argtypes = [_c_ull]
_lib.lvsa_set_wait_budget_ns.restype = _c_int
_lib.lvsa_watchdog_selftest.argtypes = [_c_ull, _c_vp]
_lib.lvsa_watchdog_selftest.restype = _c_int
_lib.lvsa_status_string.argtypes = [_c_int]
_lib.lvsa_status_string.restype = ctypes.c_char_p
_lib.lvsa_version.argtypes = []
_lib.lvsa_version.restype = _c_int


def status_string(status: int) -> str:
    return _lib.lvsa_status_string(int(status)).decode()


lvsa_status_string = status_string


def lvsa_version() -> int:
    return int(_lib.lvsa_version())


def _check(fn: str, st: int) -> None:
    if st != LVSA_OK:
        raise LvsaError(fn, st)


def lvsa_build_frame_lists(T: int, C: int, W: int, step: int, out: np.ndarray | None = None) -> np.ndarray:
    """Frame lists A(t) of step ``step`` as int32 [T, min(C, T)] (host)."""
    L = ctypes.c_int(0)
    if out is None:
        st = _lib.lvsa_build_frame_lists(T, C, W, step, None, 0, ctypes.byref(L))
        if st not in (LVSA_OK, LVSA_ERR_BUFFER_TOO_SMALL):
            _check("lvsa_build_frame_lists", st)
        out = np.empty((T, L.value), dtype=np.int32)
    if out.dtype != np.int32 or not out.flags.c_contiguous:
        raise ValueError("out must be a C-contiguous int32 array")
    st = _lib.lvsa_build_frame_lists(T, C, W, step, out.ctypes.data_as(_i32p), out.size, ctypes.byref(L))
    _check("lvsa_build_frame_lists", st)
    return out.reshape(T, L.value)


def lvsa_build_anchors(T: int, C: int, W: int, step: int) -> np.ndarray:
    """Anchor frames G_s of step ``step`` as int32 [G] (host)."""
    G = ctypes.c_int(0)
    st = _lib.lvsa_build_anchors(T, C, W, step, None, 0, ctypes.byref(G))
    if st not in (LVSA_OK, LVSA_ERR_BUFFER_TOO_SMALL):
        _check("lvsa_build_anchors", st)
    out = np.empty(G.value, dtype=np.int32)
    if G.value:
        _check("lvsa_build_anchors",
               _lib.lvsa_build_anchors(T, C, W, step, out.ctypes.data_as(_i32p), out.size, ctypes.byref(G)))
    return out


def _same_device(q, **others):
    """Every tensor of a call on q's GPU: the kernel addresses them from that device."""
    for name, x in others.items():
        if x.device != q.device:
            raise ValueError(f"{name} is on {x.device}, q on {q.device}: every tensor of a call must be on one GPU")


def _stream_ptr(stream, device):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def lvsa_attention(q, k, v, lists, tokens_per_frame: int, scale: float = 0.0, out=None, stream=None):
    """Block-sparse attention on the GPU.

    q, k, v: CUDA bf16 tensors [batch, T*tokens_per_frame, heads, d], contiguous.
    lists:   CUDA int32 tensor [T, L] of frame indices.
    Returns ``out`` (allocated with torch if not given).  Asynchronous on ``stream``
    (default: the current torch stream of q's device).
    """
    import torch

    for name, x in (("q", q), ("k", k), ("v", v)):
        if not isinstance(x, torch.Tensor) or x.device.type != "cuda" or x.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be a CUDA bfloat16 tensor")
        if not x.is_contiguous() or x.dim() != 4 or x.shape != q.shape:
            raise ValueError(f"{name} must be contiguous [batch, tokens, heads, d] shaped like q")
    if lists.device.type != "cuda" or lists.dtype != torch.int32 or lists.dim() != 2 or not lists.is_contiguous():
        raise TypeError("lists must be a contiguous CUDA int32 tensor [T, L]")
    _same_device(q, k=k, v=v, lists=lists)
    B, ntok, H, d = q.shape
    T, L = lists.shape
    if ntok != T * tokens_per_frame:
        raise ValueError(f"q has {ntok} tokens, expected T*tokens_per_frame = {T * tokens_per_frame}")
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != torch.bfloat16 or not out.is_contiguous() or out.device != q.device:
        raise ValueError("out must be a contiguous bf16 tensor shaped like q on q's device")
    with torch.cuda.device(q.device):
        st = _lib.lvsa_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), lists.data_ptr(), L, T,
                                 tokens_per_frame, H, d, B, float(scale), out.data_ptr(),
                                 _stream_ptr(stream, q.device))
    _check("lvsa_attention", st)
    return out


def lvsa_attention_joint(q, k, v, lists, tokens_per_frame: int, scale: float = 0.0, out=None, stream=None):
    """Block-sparse attention over a joint video + text sequence.

    q, k, v: CUDA bf16 [batch, T*tokens_per_frame + text_tokens, heads, d], the text tokens after the video
    (text_tokens = the tokens beyond T*tokens_per_frame).  Video rows attend their frames' lists plus every
    text token; text rows attend every token.  lists: CUDA int32 [T, L].  Returns ``out``.
    """
    import torch

    for name, x in (("q", q), ("k", k), ("v", v)):
        if not isinstance(x, torch.Tensor) or x.device.type != "cuda" or x.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be a CUDA bfloat16 tensor")
        if not x.is_contiguous() or x.dim() != 4 or x.shape != q.shape:
            raise ValueError(f"{name} must be contiguous [batch, tokens, heads, d] shaped like q")
    if lists.device.type != "cuda" or lists.dtype != torch.int32 or lists.dim() != 2 or not lists.is_contiguous():
        raise TypeError("lists must be a contiguous CUDA int32 tensor [T, L]")
    _same_device(q, k=k, v=v, lists=lists)
    B, ntok, H, d = q.shape
    T, L = lists.shape
    text = ntok - T * tokens_per_frame
    if text < 0:
        raise ValueError(f"q has {ntok} tokens, fewer than T*tokens_per_frame = {T * tokens_per_frame}")
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != torch.bfloat16 or not out.is_contiguous() or out.device != q.device:
        raise ValueError("out must be a contiguous bf16 tensor shaped like q on q's device")
    with torch.cuda.device(q.device):
        st = _lib.lvsa_attention_joint(q.data_ptr(), k.data_ptr(), v.data_ptr(), lists.data_ptr(), L, T,
                                       tokens_per_frame, text, H, d, B, float(scale), out.data_ptr(),
                                       _stream_ptr(stream, q.device))
    _check("lvsa_attention_joint", st)
    return out


def lvsa_attention_joint_raw(q_ptr: int, k_ptr: int, v_ptr: int, lists_ptr: int, L: int, T: int, P: int,
                             text: int, H: int, d: int, B: int, scale: float, out_ptr: int, stream_ptr: int) -> int:
    """The C call with raw device pointers; returns the status code unchanged."""
    return int(_lib.lvsa_attention_joint(q_ptr, k_ptr, v_ptr, lists_ptr, L, T, P, text, H, d, B, float(scale),
                                         out_ptr, ctypes.c_void_p(stream_ptr)))


def lvsa_attention_raw(q_ptr: int, k_ptr: int, v_ptr: int, lists_ptr: int, L: int, T: int, P: int, H: int,
                       d: int, B: int, scale: float, out_ptr: int, stream_ptr: int) -> int:
    """The C call with raw device pointers; returns the status code unchanged."""
    return int(_lib.lvsa_attention(q_ptr, k_ptr, v_ptr, lists_ptr, L, T, P, H, d, B, float(scale), out_ptr,
                                   ctypes.c_void_p(stream_ptr)))


def lvsa_attention_host(q_host, k_host, v_host, lists_host, tokens_per_frame: int, out_host, q_dev, k_dev, v_dev,
                        lists_dev, out_dev, scale: float = 0.0, heads_per_band: int = 0, stream=None):
    """Block-sparse attention on host tensors, uploads and readback pipelined by bands of heads.

    q_host, k_host, v_host, out_host: CPU bf16 tensors [batch, T*tokens_per_frame, heads, d], contiguous
    (pinned for overlap).  lists_host: CPU int32 [T, L].  q_dev, k_dev, v_dev, out_dev, lists_dev: CUDA
    staging tensors of the same shapes.  Asynchronous on ``stream``: synchronise it before reading out_host.
    """
    import torch

    for name, x in (("q_host", q_host), ("k_host", k_host), ("v_host", v_host), ("out_host", out_host)):
        if not isinstance(x, torch.Tensor) or x.device.type != "cpu" or x.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be a CPU bfloat16 tensor")
        if not x.is_contiguous() or x.dim() != 4 or x.shape != q_host.shape:
            raise ValueError(f"{name} must be contiguous [batch, tokens, heads, d] shaped like q_host")
    for name, x in (("q_dev", q_dev), ("k_dev", k_dev), ("v_dev", v_dev), ("out_dev", out_dev)):
        if not isinstance(x, torch.Tensor) or x.device.type != "cuda" or x.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be a CUDA bfloat16 tensor")
        if not x.is_contiguous() or x.shape != q_host.shape or x.device != q_dev.device:
            raise ValueError(f"{name} must be contiguous, shaped like q_host, on q_dev's device")
    if (lists_host.device.type != "cpu" or lists_host.dtype != torch.int32 or lists_host.dim() != 2
            or not lists_host.is_contiguous()):
        raise TypeError("lists_host must be a contiguous CPU int32 tensor [T, L]")
    if (lists_dev.device != q_dev.device or lists_dev.dtype != torch.int32 or lists_dev.shape != lists_host.shape
            or not lists_dev.is_contiguous()):
        raise TypeError("lists_dev must be a contiguous CUDA int32 tensor shaped like lists_host")
    B, ntok, H, d = q_host.shape
    T, L = lists_host.shape
    if ntok != T * tokens_per_frame:
        raise ValueError(f"q_host has {ntok} tokens, expected T*tokens_per_frame = {T * tokens_per_frame}")
    with torch.cuda.device(q_dev.device):
        st = _lib.lvsa_attention_host(q_host.data_ptr(), k_host.data_ptr(), v_host.data_ptr(), lists_host.data_ptr(),
                                      L, T, tokens_per_frame, H, d, B, float(scale), out_host.data_ptr(),
                                      q_dev.data_ptr(), k_dev.data_ptr(), v_dev.data_ptr(), lists_dev.data_ptr(),
                                      out_dev.data_ptr(), int(heads_per_band), _stream_ptr(stream, q_dev.device))
    _check("lvsa_attention_host", st)
    return out_host


def lvsa_attention_host_raw(*args) -> int:
    """The C call with raw pointers (19 arguments in the header's order); returns the status unchanged."""
    a = list(args)
    a[10] = float(a[10])
    a[18] = ctypes.c_void_p(a[18])
    return int(_lib.lvsa_attention_host(*a))


def lvsa_attention_host_static(q_host, k_host, v_host, lists_host, tokens_per_frame: int, out_host,
                               scale: float = 0.0, stream=None):
    """Block-sparse attention on host tensors with no allocation and no caller device buffer: the library
    stages everything in its own static device array (LVSA_STATIC_SCRATCH_BYTES per GPU), for callers that
    cannot allocate device memory.  q_host, k_host, v_host, out_host: CPU bf16 [batch, T*tokens_per_frame,
    heads, d], contiguous (pinned for asynchronous copies); lists_host: CPU int32 [T, L].  Runs on ``stream``
    of the current CUDA device (default: its current torch stream); synchronise before reading out_host.
    Calls that overlap on the GPU share the array and race: serialise them."""
    import torch

    for name, x in (("q_host", q_host), ("k_host", k_host), ("v_host", v_host), ("out_host", out_host)):
        if not isinstance(x, torch.Tensor) or x.device.type != "cpu" or x.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be a CPU bfloat16 tensor")
        if not x.is_contiguous() or x.dim() != 4 or x.shape != q_host.shape:
            raise ValueError(f"{name} must be contiguous [batch, tokens, heads, d] shaped like q_host")
    if (lists_host.device.type != "cpu" or lists_host.dtype != torch.int32 or lists_host.dim() != 2
            or not lists_host.is_contiguous()):
        raise TypeError("lists_host must be a contiguous CPU int32 tensor [T, L]")
    B, ntok, H, d = q_host.shape
    T, L = lists_host.shape
    if ntok != T * tokens_per_frame:
        raise ValueError(f"q_host has {ntok} tokens, expected T*tokens_per_frame = {T * tokens_per_frame}")
    dev = torch.cuda.current_device()
    st = _lib.lvsa_attention_host_static(q_host.data_ptr(), k_host.data_ptr(), v_host.data_ptr(),
                                         lists_host.data_ptr(), L, T, tokens_per_frame, H, d, B, float(scale),
                                         out_host.data_ptr(), _stream_ptr(stream, dev))
    _check("lvsa_attention_host_static", st)
    return out_host


def lvsa_attention_host_static_raw(*args) -> int:
    """The C call with raw pointers (13 arguments in the header's order); returns the status unchanged."""
    a = list(args)
    a[10] = float(a[10])
    a[12] = ctypes.c_void_p(a[12])
    return int(_lib.lvsa_attention_host_static(*a))


def _addr(x) -> int:
    """A device address: a CUDA tensor's data pointer, or an int (e.g. from lvsa_ipc_import); 0 for None."""
    if x is None:
        return 0
    return int(x.data_ptr()) if hasattr(x, "data_ptr") else int(x)


def _ptr_table(xs):
    return (ctypes.c_void_p * len(xs))(*[_addr(x) or None for x in xs])


def _int_table(xs):
    return (ctypes.c_int * len(xs))(*[int(x) for x in xs])


def lvsa_seq_to_heads_raw(q_chunks, k_chunks, v_chunks, chunk_tokens, heads: int, head0: int, band: int, d: int,
                          batch: int, q_band, k_band, v_band, stream_ptr: int = 0) -> int:
    """The C call (pointer tables as Python sequences of addresses); returns the status unchanged."""
    n = len(chunk_tokens)
    return int(_lib.lvsa_seq_to_heads(_ptr_table(q_chunks), _ptr_table(k_chunks), _ptr_table(v_chunks),
                                      _int_table(chunk_tokens), n, heads, head0, band, d, batch, _addr(q_band),
                                      _addr(k_band), _addr(v_band), ctypes.c_void_p(stream_ptr)))


def lvsa_seq_to_heads(q_chunks, k_chunks, v_chunks, chunk_tokens, head0: int, band: int, q_band, k_band, v_band,
                      heads: int | None = None, stream=None):
    """Gather heads [head0, head0 + band) of Q, K, V from token-range buffers (this GPU's tensors or peer
    addresses) into the whole-sequence band buffers q_band, k_band, v_band [batch, tokens, band, d].
    ``heads``: heads per row of the range buffers (taken from the first range that is a tensor if None)."""
    import torch

    for name, x in (("q_band", q_band), ("k_band", k_band), ("v_band", v_band)):
        if not isinstance(x, torch.Tensor) or x.device.type != "cuda" or x.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be a CUDA bfloat16 tensor")
        if not x.is_contiguous() or x.dim() != 4 or x.shape != q_band.shape:
            raise ValueError(f"{name} must be contiguous [batch, tokens, band, d] shaped like q_band")
    B, ntok, nb, d = q_band.shape
    if nb != band or ntok != sum(int(c) for c in chunk_tokens):
        raise ValueError("q_band must be [batch, sum(chunk_tokens), band, d]")
    if heads is None:
        ts = [x for x in list(q_chunks) if isinstance(x, torch.Tensor)]
        if not ts:
            raise ValueError("heads must be given when no range buffer is a tensor")
        heads = ts[0].shape[2]
    with torch.cuda.device(q_band.device):
        st = lvsa_seq_to_heads_raw(q_chunks, k_chunks, v_chunks, chunk_tokens, heads, head0, band, d, B, q_band,
                                   k_band, v_band, _stream_ptr(stream, q_band.device).value or 0)
    _check("lvsa_seq_to_heads", st)


def lvsa_attention_to_chunks_raw(q, k, v, lists, L: int, T: int, P: int, heads: int, d: int, batch: int,
                                 scale: float, out_chunks, chunk_tokens, out_heads: int, head0: int,
                                 stream_ptr: int = 0) -> int:
    """The C call (pointer tables as Python sequences of addresses); returns the status unchanged."""
    return int(_lib.lvsa_attention_to_chunks(_addr(q), _addr(k), _addr(v), _addr(lists), L, T, P, heads, d, batch,
                                             float(scale), _ptr_table(out_chunks), _int_table(chunk_tokens),
                                             len(chunk_tokens), out_heads, head0, ctypes.c_void_p(stream_ptr)))


def lvsa_attention_to_chunks(q, k, v, lists, tokens_per_frame: int, out_chunks, chunk_tokens, out_heads: int,
                             head0: int, scale: float = 0.0, stream=None):
    """Block-sparse attention of the heads of q, k, v [batch, T*P, heads, d], each output row stored into the
    token-range buffer that holds its token: out_chunks[c] [batch, chunk_tokens[c], out_heads, d] (tensors on
    this GPU or peer addresses), heads head0 .. head0 + heads - 1."""
    import torch

    for name, x in (("q", q), ("k", k), ("v", v)):
        if not isinstance(x, torch.Tensor) or x.device.type != "cuda" or x.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be a CUDA bfloat16 tensor")
        if not x.is_contiguous() or x.dim() != 4 or x.shape != q.shape:
            raise ValueError(f"{name} must be contiguous [batch, tokens, heads, d] shaped like q")
    if lists.device.type != "cuda" or lists.dtype != torch.int32 or lists.dim() != 2 or not lists.is_contiguous():
        raise TypeError("lists must be a contiguous CUDA int32 tensor [T, L]")
    _same_device(q, k=k, v=v, lists=lists)
    if len(out_chunks) != len(chunk_tokens):
        raise ValueError("one token count per output buffer")
    for x, n in zip(out_chunks, chunk_tokens):
        if isinstance(x, torch.Tensor) and (x.dtype != torch.bfloat16 or not x.is_contiguous() or x.dim() != 4
                                            or x.shape[1:] != (n, out_heads, q.shape[3])):
            raise ValueError("an output buffer tensor must be contiguous bf16 [batch, tokens of its range, "
                             "out_heads, d]")
        if isinstance(x, torch.Tensor) and x.device != q.device:
            raise ValueError("an output buffer tensor must be on q's GPU; another GPU's buffer is passed as the "
                             "address lvsa_ipc_import returned")
    B, ntok, H, d = q.shape
    T, L = lists.shape
    if ntok != T * tokens_per_frame:
        raise ValueError(f"q has {ntok} tokens, expected T*tokens_per_frame = {T * tokens_per_frame}")
    with torch.cuda.device(q.device):
        st = lvsa_attention_to_chunks_raw(q, k, v, lists, L, T, tokens_per_frame, H, d, B, scale, out_chunks,
                                          chunk_tokens, out_heads, head0,
                                          _stream_ptr(stream, q.device).value or 0)
    _check("lvsa_attention_to_chunks", st)


def lvsa_ipc_export(x) -> bytes:
    """IPC handle (LVSA_IPC_HANDLE_BYTES bytes) of the device buffer holding tensor/address ``x``."""
    buf = ctypes.create_string_buffer(LVSA_IPC_HANDLE_BYTES)
    _check("lvsa_ipc_export", _lib.lvsa_ipc_export(_addr(x), buf))
    return buf.raw


def lvsa_ipc_import(handle: bytes) -> int:
    """Maps another process's exported buffer on the current device; returns its address here."""
    if len(handle) != LVSA_IPC_HANDLE_BYTES:
        raise ValueError(f"an IPC handle has {LVSA_IPC_HANDLE_BYTES} bytes")
    ptr = ctypes.c_void_p(0)
    _check("lvsa_ipc_import", _lib.lvsa_ipc_import(ctypes.create_string_buffer(handle, len(handle)),
                                                   ctypes.byref(ptr)))
    return int(ptr.value)


def lvsa_ipc_release(ptr: int) -> None:
    _check("lvsa_ipc_release", _lib.lvsa_ipc_release(ctypes.c_void_p(int(ptr))))


def lvsa_get_device_status(clear: bool = False) -> int:
    flags = ctypes.c_uint(0)
    _check("lvsa_get_device_status", _lib.lvsa_get_device_status(ctypes.byref(flags), 1 if clear else 0))
    return int(flags.value)


def lvsa_set_wait_budget_ns(ns: int) -> None:
    _check("lvsa_set_wait_budget_ns", _lib.lvsa_set_wait_budget_ns(int(ns)))


def lvsa_watchdog_selftest(budget_ns: int, stream=None) -> None:
    import torch

    _check("lvsa_watchdog_selftest",
           _lib.lvsa_watchdog_selftest(int(budget_ns), _stream_ptr(stream, torch.cuda.current_device())))

