"""na2d_forward_host_noalloc, the host-buffer forward for callers that cannot
allocate device memory (it stages data in the library's own fixed device
array instead of a caller's workspace).

The GPU test calls it through the C ABI twice in a row -- a larger shape,
then a smaller one over the first call's leftovers in the shared array --
and checks each result against na2d_forward_host with a workspace of its
own, within the parity tolerances of the other tests.  This file is
collected last, so a run that stops at its first failure has already run
every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from vision_sliding_window_b200 import build, na2d
from vision_sliding_window_b200.inputs import make_inputs


@pytest.fixture(scope="module")
def lib():
    build.build()
    return na2d.load_library()


def test_rejects_shapes_beyond_the_fixed_array(lib):
    # 4 tensors of 2*4*256*256*32 bf16 values need 128 MiB of staging: over the 64 MiB limit
    need = lib.na2d_forward_host_workspace_bytes(2, 4, 256, 256, 32, 7, na2d.NA_BF16)
    assert need > na2d.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000)
    st = lib.na2d_forward_host_noalloc(fake, fake, fake, None, fake, 2, 4, 256, 256, 32, 7, na2d.NA_BF16, None)
    assert st == na2d.NA_ERR_UNSUPPORTED
    # argument errors are those of na2d_forward_host; an empty batch is a no-op
    assert lib.na2d_forward_host_noalloc(fake, fake, fake, None, fake, 1, 1, 8, 8, 32, 4, na2d.NA_BF16,
                                         None) == na2d.NA_ERR_INVALID_ARG
    assert lib.na2d_forward_host_noalloc(None, None, None, None, None, 0, 1, 8, 8, 32, 3, na2d.NA_BF16,
                                         None) == na2d.NA_OK


def _with_workspace(q, k, v, rpb, ks):
    out = torch.empty_like(q)
    ws = torch.empty(na2d.host_workspace_bytes(*q.shape, ks, q.dtype), dtype=torch.uint8, device="cuda")
    na2d.forward_host(q, k, v, rpb, out, ks, ws)
    torch.cuda.synchronize()
    assert na2d.device_status() == na2d.NA_OK
    return out


def _without_allocation(lib, q, k, v, rpb, ks):
    out = torch.empty_like(q)
    B, heads, H, W, d = q.shape
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.na2d_forward_host_noalloc(ptr(q), ptr(k), ptr(v), ptr(rpb), ptr(out), B, heads, H, W, d, ks,
                                       na2d._DT[q.dtype], stream)
    assert st == na2d.NA_OK, na2d.status_str(st)
    torch.cuda.synchronize()
    assert na2d.device_status() == na2d.NA_OK
    return out


@pytest.mark.gpu
def test_two_calls_match_the_workspace_entry_point(lib):
    assert torch.cuda.is_available(), "this test needs a CUDA device"
    calls = [
        ((4, 2, 40, 48, 32, 7, "bf16"), 11),  # tensor-core kernel, 15.7 MB of staging
        ((1, 1, 14, 14, 32, 7, "f32"), 12),   # SIMT kernel, over the first call's leftovers
    ]
    for (B, heads, H, W, d, ks, dt), seed in calls:
        q, k, v, rpb = make_inputs(B, heads, H, W, d, ks, dt, seed=seed)
        q, k, v, rpb = (t.pin_memory() for t in (q, k, v, rpb))
        want = _with_workspace(q, k, v, rpb, ks).double().numpy()
        got = _without_allocation(lib, q, k, v, rpb, ks).double().numpy()
        assert np.isfinite(got).all()
        if dt == "f32":
            np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-6)
        else:
            assert np.abs(got - want).max() <= 2e-2
