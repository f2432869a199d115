"""Pins of the oracle's NA over 1, 2 or 3 axes with dilation (NATTEN: NA
"from 1D to 3D"; DiNAT: dilated NA; the reading of dilation -- a query
attends within its own sub-grid of positions congruent to it mod the
dilation, with NA's clamped window there -- is stated in the oracle):

  * 2D without dilation equals the 2D NA oracle (itself pinned on its own);
  * 1D and 3D without dilation equal dense masked attention (torch fp64)
    whose windows come from an exhaustive search for the nearest window,
    not from the clamp formula;
  * dilated NA equals undilated NA run on every sub-grid (strided slices,
    of unequal lengths where the axis is not a multiple of the dilation);
  * a kernel of 1 on every axis returns v.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from tests.test_oracle_pins import brute_window_start


def rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def test_2d_equals_na2d():
    B, heads, H, W, d, ks = 2, 2, 9, 11, 8, 5
    q, k, v = (rand((B, heads, H, W, d), s) for s in (1, 2, 3))
    rpb = rand((heads, 2 * ks - 1, 2 * ks - 1), 4, 0.5)
    np.testing.assert_allclose(oracle.nd_forward(q, k, v, rpb, (ks, ks)), oracle.forward(q, k, v, rpb, ks),
                               rtol=1e-12, atol=1e-12)


def dense_nd(q, k, v, rpb, ks):
    """Full attention over every position with a -inf mask outside each
    query's window (nearest window by exhaustive search on each axis) and
    the bias gathered by displacement; torch fp64."""
    B, heads, *L, d = q.shape
    grids = []
    for La, ka in zip(L, ks):
        st = torch.tensor([brute_window_start(i, La, ka) for i in range(La)])
        pos = torch.arange(La)
        inside = (pos[None, :] >= st[:, None]) & (pos[None, :] < st[:, None] + ka)  # [query, key]
        disp = (pos[None, :] - torch.arange(La)[:, None] + ka - 1).clamp(0, 2 * ka - 2)
        grids.append((inside, disp))
    n = int(np.prod(L))
    mask = torch.ones((n, n), dtype=torch.bool)
    bias = torch.zeros((heads, n, n), dtype=torch.float64)
    qi = list(itertools.product(*[range(La) for La in L]))
    for a, qa in enumerate(qi):
        for b, kb in enumerate(qi):
            ok = all(bool(g[0][qa[t], kb[t]]) for t, g in enumerate(grids))
            mask[a, b] = ok
            if ok and rpb is not None:
                idx = tuple(int(g[1][qa[t], kb[t]]) for t, g in enumerate(grids))
                bias[:, a, b] = torch.tensor(rpb[(slice(None),) + idx])
    Q, K, V = (torch.tensor(x).reshape(B, heads, n, d) for x in (q, k, v))
    logits = (Q @ K.transpose(-1, -2) + bias[None]).masked_fill(~mask, float("-inf"))
    return (torch.softmax(logits / math.sqrt(d), -1) @ V).reshape(q.shape).numpy()


@pytest.mark.parametrize("L,ks", [((13,), (5,)), ((9,), (3,)), ((4, 5, 6), (3, 3, 5)), ((5, 3, 4), (5, 1, 3))])
def test_1d_and_3d_equal_dense_masked_attention(L, ks):
    B, heads, d = 2, 2, 4
    q, k, v = (rand((B, heads, *L, d), s) for s in (5, 6, 7))
    rpb = rand((heads, *[2 * ka - 1 for ka in ks]), 8, 0.5)
    np.testing.assert_allclose(oracle.nd_forward(q, k, v, rpb, ks), dense_nd(q, k, v, rpb, ks),
                               rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("L,ks,dil", [((14, 13), (3, 5), (2, 2)), ((20,), (5,), (3,)), ((7, 9, 10), (3, 3, 3), (1, 2, 3)),
                                      ((12, 12), (5, 3), (2, 1))])
def test_dilation_is_na_on_every_sub_grid(L, ks, dil):
    B, heads, d = 1, 2, 4
    q, k, v = (rand((B, heads, *L, d), s) for s in (9, 10, 11))
    rpb = rand((heads, *[2 * ka - 1 for ka in ks]), 12, 0.5)
    got = oracle.nd_forward(q, k, v, rpb, ks, dil)
    want = np.empty_like(got)
    for res in itertools.product(*[range(da) for da in dil]):
        sl = (slice(None), slice(None)) + tuple(slice(r, None, da) for r, da in zip(res, dil)) + (slice(None),)
        want[sl] = oracle.nd_forward(q[sl], k[sl], v[sl], rpb, ks)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_unit_kernel_returns_values():
    q, k, v = (rand((2, 3, 4, 5, 6, 8), s) for s in (13, 14, 15))
    np.testing.assert_allclose(oracle.nd_forward(q, k, v, rand((3, 1, 1, 1), 16), (1, 1, 1), (2, 1, 3)), v,
                               rtol=0, atol=1e-15)
