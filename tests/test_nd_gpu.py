"""Parity of na_forward_nd (through the C ABI) with the oracle's NA over 1-3
axes with dilation, on the same seeded inputs; tolerances as for the
forward (float32 rtol 1e-5 / atol 1e-6, 16-bit max-abs 2e-2)."""
import numpy as np
import pytest
import torch

import oracle
from vision_sliding_window_b200 import build, na2d
from vision_sliding_window_b200.inputs import DTYPES

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    build.build()
    return na2d.load_library()


CASES = [
    # spatial, ks, dilation, d, dtype
    ((61,), (7,), (1,), 32, "f32"),
    ((257,), (13,), (3,), 64, "bf16"),
    ((96,), (5,), (4,), 16, "f16"),
    ((24, 30), (7, 5), (2, 3), 32, "bf16"),
    ((56, 56), (7, 7), (1, 1), 32, "f32"),
    ((40, 36), (5, 5), (4, 2), 64, "f16"),
    ((8, 12, 10), (3, 5, 3), (1, 2, 3), 32, "bf16"),
    ((6, 9, 9), (5, 3, 3), (1, 1, 1), 16, "f32"),
    ((12, 10, 8), (3, 3, 3), (2, 2, 2), 128, "f16"),
]


@pytest.mark.parametrize("spatial,ks,dil,d,dtype", CASES)
def test_nd_matches_oracle(spatial, ks, dil, d, dtype):
    B, heads = 2, 2
    g = torch.Generator().manual_seed(sum(spatial) + sum(ks))
    q, k, v = (torch.randn((B, heads, *spatial, d), generator=g).to(DTYPES[dtype]) for _ in range(3))
    rpb = (torch.randn((heads, *[2 * ka - 1 for ka in ks]), generator=g) * 0.5).to(DTYPES[dtype])
    out = na2d.forward_nd(*(t.cuda() for t in (q, k, v, rpb)), ks, dil)
    torch.cuda.synchronize()
    want = oracle.nd_forward(q, k, v, rpb, ks, dil)
    got = out.double().cpu().numpy()
    assert np.isfinite(got).all()
    if dtype == "f32":
        np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-6)
    else:
        assert np.abs(got - want).max() <= 2e-2, np.abs(got - want).max()


def test_2d_without_dilation_matches_the_fused_forward():
    q, k, v = (torch.randn((2, 2, 40, 48, 32), generator=torch.Generator().manual_seed(s)).to(torch.bfloat16)
               for s in (1, 2, 3))
    rpb = (torch.randn((2, 13, 13), generator=torch.Generator().manual_seed(4)) * 0.5).to(torch.bfloat16)
    dev = [t.cuda() for t in (q, k, v, rpb)]
    a = na2d.forward_nd(*dev, (7, 7)).float()
    b = na2d.forward(*dev, 7).float()
    torch.cuda.synchronize()
    assert (a - b).abs().max().item() <= 2e-2
