"""Pins of the oracle's SASA (stand-alone self-attention: the centred window
with zero padding; NAT Sec. 3.2 calls it NA on a zero-padded input; the
Qiita SASA/NA drawing shows the two windows at the borders):

  * the pages' own statement, as an identity: SASA of a map equals the NA
    oracle run on the map zero-padded by k/2 on every side, at the original
    pixels (the NA oracle is independent code, pinned on its own);
  * an independent dense formulation (torch fp64): attention over every
    position of the padded map with a -inf mask outside each query's centred
    window, the bias gathered by displacement;
  * queries whose centred window lies inside the map give NA's output;
  * k = 1 gives v; the drawing's geometry: on a row of 5 with k = 3 the
    border queries reach one position into the padding.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from vision_sliding_window_b200.inputs import make_inputs


def f64(*ts):
    return [None if t is None else t.double().numpy() for t in ts]


CASES = [(1, 2, 9, 11, 8, 3, True), (2, 1, 7, 7, 4, 7, True), (1, 2, 12, 10, 16, 5, False), (1, 1, 5, 13, 4, 5, True)]


@pytest.mark.parametrize("B,heads,H,W,d,ks,with_rpb", CASES)
def test_sasa_equals_na_on_the_zero_padded_map(B, heads, H, W, d, ks, with_rpb):
    q, k, v, rpb = f64(*make_inputs(B, heads, H, W, d, ks, "f32", seed=H + ks, rpb_std=0.5, with_rpb=with_rpb))
    p = ks // 2
    pad = lambda x: np.pad(x, ((0, 0), (0, 0), (p, p), (p, p), (0, 0)))
    want = oracle.forward(pad(q), pad(k), pad(v), rpb, ks)[:, :, p:p + H, p:p + W]
    np.testing.assert_allclose(oracle.sasa_forward(q, k, v, rpb, ks), want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("B,heads,H,W,d,ks,with_rpb", CASES)
def test_sasa_equals_dense_masked_attention_with_zero_padding(B, heads, H, W, d, ks, with_rpb):
    q, k, v, rpb = f64(*make_inputs(B, heads, H, W, d, ks, "f32", seed=2 * H + ks, rpb_std=0.5,
                                    with_rpb=with_rpb))
    p = ks // 2
    Hp, Wp = H + 2 * p, W + 2 * p
    kp = torch.zeros((B, heads, Hp, Wp, d), dtype=torch.float64)
    vp = torch.zeros_like(kp)
    kp[:, :, p:p + H, p:p + W] = torch.tensor(k)
    vp[:, :, p:p + H, p:p + W] = torch.tensor(v)
    qi = torch.tensor(q)
    # query (i, j) sits at padded (i + p, j + p); its window is padded rows [i, i + ks), columns [j, j + ks)
    ri, rr = torch.arange(H)[:, None], torch.arange(Hp)[None, :]
    ci, cc = torch.arange(W)[:, None], torch.arange(Wp)[None, :]
    in_r = (rr >= ri) & (rr < ri + ks)
    in_c = (cc >= ci) & (cc < ci + ks)
    mask = in_r[:, None, :, None] & in_c[None, :, None, :]  # [i, j, r, t]
    logits = torch.einsum("bhijx,bhrtx->bhijrt", qi, kp)
    if with_rpb:
        dr = (rr - (ri + p) + ks - 1).clamp(0, 2 * ks - 2)
        dc = (cc - (ci + p) + ks - 1).clamp(0, 2 * ks - 2)
        logits = logits + torch.tensor(rpb)[:, dr[:, None, :, None], dc[None, :, None, :]][None]
    logits = logits.masked_fill(~mask, float("-inf")).reshape(B, heads, H, W, Hp * Wp)
    prob = torch.softmax(logits / math.sqrt(d), dim=-1)
    want = torch.einsum("bhijn,bhnx->bhijx", prob, vp.reshape(B, heads, Hp * Wp, d)).numpy()
    np.testing.assert_allclose(oracle.sasa_forward(q, k, v, rpb, ks), want, rtol=1e-10, atol=1e-12)


def test_sasa_equals_na_where_the_window_is_inside_the_map():
    B, heads, H, W, d, ks = 1, 2, 15, 14, 8, 5
    q, k, v, rpb = f64(*make_inputs(B, heads, H, W, d, ks, "f32", seed=5, rpb_std=0.5))
    s, n = oracle.sasa_forward(q, k, v, rpb, ks), oracle.forward(q, k, v, rpb, ks)
    p = ks // 2
    np.testing.assert_allclose(s[:, :, p:H - p, p:W - p], n[:, :, p:H - p, p:W - p], rtol=1e-12, atol=1e-12)
    assert np.abs(s[:, :, 0, 0] - n[:, :, 0, 0]).max() > 1e-3  # and differs at the corner


def test_sasa_k1_is_identity_and_border_reaches_into_padding():
    q, k, v, rpb = f64(*make_inputs(2, 2, 6, 7, 8, 1, "f32", seed=6, rpb_std=1.0))
    np.testing.assert_allclose(oracle.sasa_forward(q, k, v, rpb, 1), v, rtol=0, atol=1e-15)
    # a row of 5 pixels, k = 3: only the padding's zero value and its bias reach the first query
    q, k, v, rpb = f64(*make_inputs(1, 1, 3, 5, 4, 3, "f32", seed=7, rpb_std=0.0))
    q[:] = 0.0
    out = oracle.sasa_forward(q, k, v, None, 3)
    # with q = 0 and no bias every window entry weighs 1/9; zero padding lowers the corner's mean
    np.testing.assert_allclose(out[0, 0, 0, 0], v[0, 0, 0:2, 0:2].sum(axis=(0, 1)) / 9, rtol=1e-12)
