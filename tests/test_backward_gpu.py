"""Parity of na2d_backward (through the C ABI) with the fp64 oracle's
backward on the same seeded inputs and the same upstream gradient.

Tolerances: float32 inputs -- |gpu - oracle| <= 1e-6 + 1e-5 |oracle|
elementwise (float64 accumulation on the GPU); fp16 / bf16 inputs with
float32 accumulation -- max |gpu - oracle| <= 2e-2 * max(1, max |oracle|) for
each gradient, the forward's 16-bit bound scaled to the gradient's size
(gradients are sums of up to k^2 terms and can exceed 1).  The float32 bias
gradient of 16-bit inputs uses the same scaled bound.
"""
import numpy as np
import pytest
import torch

import oracle
from vision_sliding_window_b200 import build, na2d
from vision_sliding_window_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    build.build()
    return na2d.load_library()


def check(got, want, dtype, what):
    g = got.detach().double().cpu().numpy()
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    if dtype == "f32":
        np.testing.assert_allclose(g, want, rtol=1e-5, atol=1e-6, err_msg=what)
    else:
        bound = 2e-2 * max(1.0, float(np.abs(want).max()))
        err = float(np.abs(g - want).max())
        assert err <= bound, f"{what}: max abs error {err:.3e} > {bound:.3e}"


CASES = [
    # B, heads, H, W, d, ks, dtype, with_rpb
    (1, 1, 14, 14, 32, 7, "f32", True),
    (2, 2, 9, 11, 16, 3, "f32", True),
    (1, 2, 13, 12, 64, 11, "f32", False),
    (2, 2, 24, 20, 32, 7, "bf16", True),
    (2, 3, 17, 23, 64, 5, "f16", True),
    (1, 2, 30, 28, 32, 13, "bf16", True),
    (1, 1, 7, 7, 32, 7, "f16", True),      # k = H = W
    (2, 1, 10, 9, 128, 9, "bf16", False),
    (1, 2, 6, 8, 32, 1, "bf16", True),     # k = 1
]


@pytest.mark.parametrize("B,heads,H,W,d,ks,dtype,with_rpb", CASES)
def test_backward_matches_oracle(B, heads, H, W, d, ks, dtype, with_rpb):
    q, k, v, rpb = make_inputs(B, heads, H, W, d, ks, dtype, seed=B * 100 + H + ks, rpb_std=0.5,
                               with_rpb=with_rpb)
    g = torch.Generator().manual_seed(ks + 7)
    dout = torch.randn(q.shape, generator=g).to(q.dtype)
    dev = [None if t is None else t.cuda() for t in (q, k, v, rpb, dout)]
    dq, dk, dv, drpb = na2d.backward(*dev, ks)
    torch.cuda.synchronize()
    assert na2d.device_status() == na2d.NA_OK
    want = oracle.backward(q, k, v, rpb, dout, ks)
    for name, got, w in zip(("dq", "dk", "dv"), (dq, dk, dv), want[:3]):
        check(got, w, dtype, name)
    if with_rpb:
        check(drpb, want[3], dtype, "drpb")
    else:
        # the gradient with respect to a zero bias: the oracle's, with a zero table
        zero = torch.zeros((heads, 2 * ks - 1, 2 * ks - 1), dtype=q.dtype)
        check(drpb, oracle.backward(q, k, v, zero, dout, ks)[3], dtype, "drpb (zero bias)")


def test_backward_of_a_workload_sized_map_at_sampled_keys():
    """Stage-1 shape (32x2x56x56, d=32, k=7, bf16): every gradient compared with
    the oracle on the first and last (b, h) map (the backward of one map is
    independent of the others, except the bias gradient, compared in full)."""
    B, heads, H, W, d, ks = 32, 2, 56, 56, 32, 7
    q, k, v, rpb = make_inputs(B, heads, H, W, d, ks, "bf16", seed=0)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(1)).to(q.dtype)
    dq, dk, dv, drpb = na2d.backward(*(t.cuda() for t in (q, k, v, rpb, dout)), ks)
    torch.cuda.synchronize()
    assert na2d.device_status() == na2d.NA_OK
    for b, h in ((0, 0), (B - 1, heads - 1)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        want = oracle.backward(q[sl], k[sl], v[sl], rpb[h:h + 1], dout[sl], ks)
        for name, got, w in zip(("dq", "dk", "dv"), (dq, dk, dv), want[:3]):
            check(got[sl], w, "bf16", f"{name} map ({b},{h})")
    check(drpb, oracle.backward(q, k, v, rpb, dout, ks)[3], "bf16", "drpb")


def test_backward_writes_exactly_its_outputs():
    shp = (2, 2, 15, 17, 32)
    q, k, v, rpb = make_inputs(*shp, 5, "bf16", seed=9)
    dout = torch.randn(shp, generator=torch.Generator().manual_seed(2)).to(q.dtype)
    bufs = []
    outs = []
    for _ in range(3):
        buf = torch.full((int(np.prod(shp)) + 2 * 4096,), float("nan"), dtype=q.dtype, device="cuda")
        bufs.append(buf)
        outs.append(buf[4096:-4096].view(shp))
    dq, dk, dv = outs
    drpb = torch.full((2, 9, 9), float("nan"), dtype=torch.float32, device="cuda")
    lib = na2d.load_library()
    import ctypes
    ws = torch.empty(lib.na2d_backward_workspace_bytes(*shp, 5, na2d.NA_BF16), dtype=torch.uint8, device="cuda")
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    dev = [t.cuda() for t in (q, k, v, rpb, dout)]
    st = lib.na2d_backward(*(P(t) for t in dev), P(dq), P(dk), P(dv), P(drpb), P(ws), ws.numel(), *shp, 5,
                           na2d.NA_BF16, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == na2d.NA_OK
    torch.cuda.synchronize()
    for buf, o in zip(bufs, outs):
        assert torch.isfinite(o).all()
        assert torch.isnan(buf[:4096]).all() and torch.isnan(buf[-4096:]).all()
    assert torch.isfinite(drpb).all()
