"""Parity of na2d_block_forward (through the C ABI) with the oracle's NA
block on the same seeded inputs.  The oracle rounds q, k, v and the
attention output to the input dtype where the GPU stores them; bounds:
float32 rtol 1e-5 / atol 1e-5 (cuBLAS sums the projections in float32 in
its own order), 16-bit max-abs 2e-2."""
import numpy as np
import pytest
import torch

import oracle
from vision_sliding_window_b200 import build, na2d
from vision_sliding_window_b200.inputs import make_block_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    build.build()
    return na2d.load_library()


CASES = [
    # B, H, W, heads, dh, ks, dtype, biases
    (2, 14, 14, 2, 32, 7, "f32", True),
    (4, 28, 28, 2, 32, 7, "bf16", True),
    (2, 30, 26, 3, 64, 5, "f16", True),
    (1, 40, 36, 4, 32, 13, "bf16", False),
    (2, 9, 11, 4, 16, 3, "f16", True),
]


@pytest.mark.parametrize("B,H,W,heads,dh,ks,dtype,biases", CASES)
def test_block_matches_oracle(B, H, W, heads, dh, ks, dtype, biases):
    x, wqkv, bqkv, wo, bo, rpb = make_block_inputs(B, H, W, heads, dh, ks, dtype, seed=H + ks)
    if not biases:
        bqkv = bo = None
    dev = [None if t is None else t.cuda() for t in (x, wqkv, bqkv, wo, bo, rpb)]
    y = na2d.block_forward(*dev, heads, ks)
    torch.cuda.synchronize()
    assert na2d.device_status() == na2d.NA_OK
    want = oracle.block_forward(x, wqkv, bqkv, wo, bo, rpb, heads, ks, store=None if dtype == "f32" else dtype)
    got = y.double().cpu().numpy()
    assert np.isfinite(got).all()
    if dtype == "f32":
        np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-5)
    else:
        assert np.abs(got - want).max() <= 2e-2, np.abs(got - want).max()
