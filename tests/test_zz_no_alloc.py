"""The allocation-free host-buffer call (lvsa_attention_host_static) against the host-buffer call that uses
caller staging buffers (lvsa_attention_host), through the C ABI.

Some callers cannot allocate device memory: a plug-in inside a process whose allocator already owns the GPU's
memory, or code on a path where cudaMalloc / cudaFree must not run because they can block or synchronise the
device.  For them the library stages everything in its own static device array.  This file runs last (the
name sorts last), and also passes on its own in a fresh process: its first call sets the array up.
"""

import pytest
import torch

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def pinned_inputs(T, P, H, d, B, seed):
    g = torch.Generator().manual_seed(seed)
    xs = [torch.randn((B, T * P, H, d), generator=g).to(torch.bfloat16).pin_memory() for _ in range(3)]
    return xs


def with_staging_buffers(lib, q, k, v, lists, P):
    """The existing host-buffer call, staging in device buffers the caller allocates."""
    out = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    stage = [torch.empty(q.shape, dtype=torch.bfloat16, device="cuda") for _ in range(4)]
    lists_dev = torch.empty(lists.shape, dtype=torch.int32, device="cuda")
    lib.lvsa_attention_host(q, k, v, lists, P, out, stage[0], stage[1], stage[2], lists_dev, stage[3])
    torch.cuda.synchronize()
    return out


def without_allocation(lib, q, k, v, lists, P):
    """The allocation-free call through the C ABI (raw pointers), on the current stream."""
    out = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    B, ntok, H, d = q.shape
    T, L = lists.shape
    st = lib.lvsa_attention_host_static_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), lists.data_ptr(), L, T, P, H,
                                            d, B, 0.0, out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == lib.LVSA_OK, lib.status_string(st)
    torch.cuda.synchronize()
    return out


def test_static_staging_matches_caller_staging_on_two_calls_in_a_row(gpu_lib):
    # the second call is smaller and uses other inputs and lists: whatever the first call left in the shared
    # array beyond the second call's extent must not leak into its result
    cases = [(6, 300, 3, 128, 2, 3, 1, 4, 11), (8, 64, 2, 64, 1, 4, 2, 5, 12)]
    for T, P, H, d, B, C, W, step, seed in cases:
        q, k, v = pinned_inputs(T, P, H, d, B, seed)
        lists = torch.from_numpy(gpu_lib.lvsa_build_frame_lists(T, C, W, step)).pin_memory()
        ref = with_staging_buffers(gpu_lib, q, k, v, lists, P)
        got = without_allocation(gpu_lib, q, k, v, lists, P)
        err = (got.float() - ref.float()).abs()
        assert torch.isfinite(got.float()).all()
        assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS, (T, P, err.max().item())
    assert gpu_lib.lvsa_get_device_status(clear=True) == 0


def test_static_staging_size_limit(gpu_lib):
    """Q, K, V and the output (each rounded up to 256 bytes) plus the lists must fit in the array: one frame
    more than fits is refused before any copy or launch; the largest call that fits runs and matches."""
    A = 1 << 24  # fake host addresses for the refused call: the size check comes before anything else
    n = 1 << 26
    P, H, d, C, W = 2048, 1, 128, 7, 3      # 512 KiB per frame and tensor
    T = 32                                   # 4 x 16 MiB = the whole array, no room left for the lists
    st = gpu_lib.lvsa_attention_host_static_raw(A, A + n, A + 2 * n, A + 3 * n, C, T, P, H, d, 1, 0.0, A + 4 * n, 0)
    assert st == gpu_lib.LVSA_ERR_INVALID_ARG
    T = 31                                   # 4 x 15.5 MiB + the lists: fits
    assert 4 * T * P * H * d * 2 + 256 <= gpu_lib.LVSA_STATIC_SCRATCH_BYTES
    q, k, v = pinned_inputs(T, P, H, d, 1, 13)
    lists = torch.from_numpy(gpu_lib.lvsa_build_frame_lists(T, C, W, 9)).pin_memory()
    ref = with_staging_buffers(gpu_lib, q, k, v, lists, P)
    got = without_allocation(gpu_lib, q, k, v, lists, P)
    err = (got.float() - ref.float()).abs()
    assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS
