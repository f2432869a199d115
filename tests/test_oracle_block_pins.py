"""Pins of the oracle's NA block (NAT App. A.1: Q/K/V projections, NA, an
output projection):

  * identity projections (q = k = v = x, Wo = I, no biases) reduce the block
    to the NA oracle on x split into heads;
  * an independent torch fp64 composition (einsum projections around dense
    masked attention) agrees to 1e-10;
  * the output projection is affine: y(2 Wo, 2 bo) = 2 y(Wo, bo);
  * rounding q, k, v, o and y to 16 bits moves y by a small multiple of the
    type's spacing, and by more than nothing.

tests/test_oracle_mutations.py plants mistakes in a copy of the block and
checks that one of these fails.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.test_oracle_backward_pins import dense_masked_attention_torch


def block_inputs(B, H, W, heads, dh, ks, seed):
    g = torch.Generator().manual_seed(seed)
    C = heads * dh
    x = torch.randn((B, H, W, C), generator=g, dtype=torch.float64)
    wqkv = torch.randn((C, 3 * C), generator=g, dtype=torch.float64) / math.sqrt(C)
    bqkv = torch.randn(3 * C, generator=g, dtype=torch.float64) * 0.1
    wo = torch.randn((C, C), generator=g, dtype=torch.float64) / math.sqrt(C)
    bo = torch.randn(C, generator=g, dtype=torch.float64) * 0.1
    rpb = torch.randn((heads, 2 * ks - 1, 2 * ks - 1), generator=g, dtype=torch.float64) * 0.5
    return [t.numpy() for t in (x, wqkv, bqkv, wo, bo, rpb)]


def test_identity_projections_reduce_to_na():
    B, H, W, heads, dh, ks = 2, 9, 8, 2, 8, 5
    x, _, _, _, _, rpb = block_inputs(B, H, W, heads, dh, ks, 1)
    C = heads * dh
    eye = np.eye(C)
    y = oracle.block_forward(x, np.concatenate([eye, eye, eye], axis=1), None, eye, None, rpb, heads, ks)
    xh = np.ascontiguousarray(x.reshape(B, H, W, heads, dh).transpose(0, 3, 1, 2, 4))
    want = oracle.forward(xh, xh, xh, rpb, ks).transpose(0, 2, 3, 1, 4).reshape(B, H, W, C)
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("B,H,W,heads,dh,ks", [(1, 7, 9, 2, 8, 3), (2, 8, 8, 3, 4, 5), (1, 6, 6, 1, 16, 5)])
def test_block_equals_independent_torch_composition(B, H, W, heads, dh, ks):
    x, wqkv, bqkv, wo, bo, rpb = block_inputs(B, H, W, heads, dh, ks, B + H + ks)
    C = heads * dh
    tx, tw, tb, two, tbo, trpb = (torch.tensor(a) for a in (x, wqkv, bqkv, wo, bo, rpb))
    qkv = torch.einsum("bhwc,cn->bhwn", tx, tw) + tb
    q, k, v = (qkv[..., s * C:(s + 1) * C].reshape(B, H, W, heads, dh).permute(0, 3, 1, 2, 4) for s in range(3))
    o = dense_masked_attention_torch(q, k, v, trpb, ks).permute(0, 2, 3, 1, 4).reshape(B, H, W, C)
    want = (torch.einsum("bhwc,cn->bhwn", o, two) + tbo).numpy()
    np.testing.assert_allclose(oracle.block_forward(x, wqkv, bqkv, wo, bo, rpb, heads, ks), want,
                               rtol=1e-10, atol=1e-12)


def test_output_projection_is_affine():
    x, wqkv, bqkv, wo, bo, rpb = block_inputs(1, 7, 7, 2, 8, 3, 9)
    y1 = oracle.block_forward(x, wqkv, bqkv, wo, bo, rpb, 2, 3)
    y2 = oracle.block_forward(x, wqkv, bqkv, 2 * wo, 2 * bo, rpb, 2, 3)
    np.testing.assert_allclose(y2, 2 * y1, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("store", ["bf16", "f16"])
def test_storage_rounding_stays_within_its_bound(store):
    x, wqkv, bqkv, wo, bo, rpb = block_inputs(2, 8, 9, 2, 16, 5, 11)
    exact = oracle.block_forward(x, wqkv, bqkv, wo, bo, rpb, 2, 5)
    rounded = oracle.block_forward(x, wqkv, bqkv, wo, bo, rpb, 2, 5, store=store)
    err = np.abs(rounded - exact).max()
    eps = 2.0 ** -8 if store == "bf16" else 2.0 ** -11
    assert 0 < err < 30 * eps * max(1.0, np.abs(exact).max())
