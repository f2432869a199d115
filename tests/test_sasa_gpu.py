"""Parity of na2d_sasa_forward (through the C ABI) with the oracle's SASA on
the same seeded inputs: every element on small maps, including windows
larger than the map, and sampled rows of a workload-sized map.  Tolerances
as for the forward: float32 rtol 1e-5 / atol 1e-6; 16-bit max-abs 2e-2."""
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
        err = float(np.abs(g - want).max())
        assert err <= 2e-2, f"{what}: max abs error {err:.3e}"


CASES = [
    # B, heads, H, W, d, ks, dtype, rpb
    (1, 1, 14, 14, 32, 7, "f32", True),
    (2, 2, 24, 20, 32, 7, "bf16", True),
    (2, 3, 17, 23, 64, 5, "f16", True),
    (1, 2, 30, 28, 32, 13, "bf16", True),
    (2, 2, 9, 11, 16, 3, "f16", False),
    (1, 2, 5, 6, 32, 7, "bf16", True),      # window larger than the map
    (1, 1, 7, 7, 64, 9, "f16", True),       # window larger than the map
    (2, 1, 10, 9, 128, 1, "bf16", True),    # k = 1
]


@pytest.mark.parametrize("B,heads,H,W,d,ks,dtype,with_rpb", CASES)
def test_sasa_matches_oracle(B, heads, H, W, d, ks, dtype, with_rpb):
    q, k, v, rpb = make_inputs(B, heads, H, W, d, ks, dtype, seed=B * 7 + H + ks, rpb_std=0.5,
                               with_rpb=with_rpb)
    out = na2d.sasa_forward(*[None if t is None else t.cuda() for t in (q, k, v, rpb)], ks)
    torch.cuda.synchronize()
    assert na2d.device_status() == na2d.NA_OK
    check(out, oracle.sasa_forward(q, k, v, rpb, ks), dtype, "sasa")


def test_sasa_of_a_stage1_map():
    """Stage-1 shape (32x2x56x56, d=32, k=7, bf16): the first and last map in full."""
    B, heads, H, W, d, ks = 32, 2, 56, 56, 32, 7
    q, k, v, rpb = make_inputs(B, heads, H, W, d, ks, "bf16", seed=0)
    out = na2d.sasa_forward(*(t.cuda() for t in (q, k, v, rpb)), ks).cpu()
    for b, h in ((0, 0), (B - 1, heads - 1)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        want = oracle.sasa_forward(q[sl], k[sl], v[sl], rpb[h:h + 1], ks)
        check(out[sl], want, "bf16", f"map ({b},{h})")
