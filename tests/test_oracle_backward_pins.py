"""Pins of the oracle's backward pass (the gradients of Eqs. (2)-(4) that
NATTEN provides for "QK+B" and "AV") to what the mathematics fixes:

  * central finite differences of the oracle's own forward on tiny maps --
    the gradient's definition, independent of the hand-derived chain rule;
  * torch fp64 autograd through an independent dense formulation (full
    attention over all H*W keys with a -inf mask outside each query's
    window and the bias gathered from the table by displacement);
  * closed forms: k = 1 (one key per query: dv = dout, everything else 0),
    constant values (dP is constant over the window, so the softmax Jacobian
    kills dq, dk and the bias gradient; dv = sum of P * dout);
  * an invariant: each query's logit gradients sum to zero (the softmax
    Jacobian's rows sum to zero), so every head's bias gradient sums to 0.

tests/test_oracle_mutations.py plants mistakes in the backward and checks
that one of these fails.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.test_oracle_pins import brute_window_start
from vision_sliding_window_b200.inputs import make_inputs


def f64(*ts):
    return [None if t is None else np.asarray(t.double().numpy() if torch.is_tensor(t) else t, dtype=np.float64)
            for t in ts]


def case(B, heads, H, W, d, ks, seed, with_rpb=True, rpb_std=0.5):
    q, k, v, rpb = f64(*make_inputs(B, heads, H, W, d, ks, "f32", seed=seed, rpb_std=rpb_std, with_rpb=with_rpb))
    dout = np.random.default_rng(seed + 99).standard_normal(q.shape)
    return q, k, v, rpb, dout


def loss(q, k, v, rpb, dout, ks):
    return float((oracle.forward(q, k, v, rpb, ks, nthreads=1) * dout).sum())


FD_CASES = [
    (1, 2, 5, 6, 4, 3, True),
    (2, 1, 7, 5, 3, 5, True),
    (1, 1, 4, 4, 2, 3, False),
    (1, 1, 6, 6, 3, 5, True),
]


@pytest.mark.parametrize("B,heads,H,W,d,ks,with_rpb", FD_CASES)
def test_backward_matches_central_differences(B, heads, H, W, d, ks, with_rpb):
    q, k, v, rpb, dout = case(B, heads, H, W, d, ks, seed=H * 10 + ks, with_rpb=with_rpb)
    grads = oracle.backward(q, k, v, rpb, dout, ks, nthreads=1)
    eps = 1e-5
    args = [q, k, v, rpb]
    for which in range(4 if with_rpb else 3):
        x = args[which]
        num = np.empty_like(x)
        for idx in np.ndindex(*x.shape):
            keep = x[idx]
            x[idx] = keep + eps
            up = loss(*args, dout, ks)
            x[idx] = keep - eps
            down = loss(*args, dout, ks)
            x[idx] = keep
            num[idx] = (up - down) / (2 * eps)
        np.testing.assert_allclose(grads[which], num, rtol=1e-6, atol=1e-8,
                                   err_msg=f"gradient {'q k v rpb'.split()[which]}")
    if not with_rpb:
        assert grads[3] is None


def dense_masked_attention_torch(q, k, v, rpb, ks):
    """Full self-attention over all H*W keys with a -inf mask outside each
    query's window (found by exhaustive search, not the clamp formula) and
    the bias gathered by displacement; torch fp64, differentiable."""
    B, heads, H, W, d = q.shape
    sr = torch.tensor([brute_window_start(i, H, ks) for i in range(H)])
    sc = torch.tensor([brute_window_start(j, W, ks) for j in range(W)])
    rr, tt = torch.arange(H), torch.arange(W)
    in_r = (rr[None, :] >= sr[:, None]) & (rr[None, :] < sr[:, None] + ks)
    in_c = (tt[None, :] >= sc[:, None]) & (tt[None, :] < sc[:, None] + ks)
    mask = in_r[:, None, :, None] & in_c[None, :, None, :]  # [i, j, r, t]
    dr = (rr[None, :] - rr[:, None] + ks - 1).clamp(0, 2 * ks - 2)
    dc = (tt[None, :] - tt[:, None] + ks - 1).clamp(0, 2 * ks - 2)
    logits = torch.einsum("bhijx,bhrtx->bhijrt", q, k)
    if rpb is not None:
        logits = logits + rpb[:, dr[:, None, :, None], dc[None, :, None, :]][None]
    logits = logits.masked_fill(~mask, float("-inf")).reshape(B, heads, H, W, H * W)
    p = torch.softmax(logits / math.sqrt(d), dim=-1)
    return torch.einsum("bhijn,bhnx->bhijx", p, v.reshape(B, heads, H * W, d))


AUTOGRAD_CASES = [
    (2, 2, 9, 11, 8, 3, True),
    (1, 3, 8, 8, 16, 7, True),
    (2, 1, 7, 7, 4, 7, True),   # k = H = W: plain self-attention
    (1, 2, 10, 6, 5, 5, False),
    (1, 1, 13, 12, 4, 11, True),
]


@pytest.mark.parametrize("B,heads,H,W,d,ks,with_rpb", AUTOGRAD_CASES)
def test_backward_equals_autograd_of_dense_masked_attention(B, heads, H, W, d, ks, with_rpb):
    q, k, v, rpb, dout = case(B, heads, H, W, d, ks, seed=B + H + ks, with_rpb=with_rpb)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    trpb = torch.tensor(rpb, requires_grad=True) if with_rpb else None
    out = dense_masked_attention_torch(tq, tk, tv, trpb, ks)
    (out * torch.tensor(dout)).sum().backward()
    dq, dk, dv, drpb = oracle.backward(q, k, v, rpb, dout, ks)
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-10, atol=1e-12)
    if with_rpb:
        np.testing.assert_allclose(drpb, trpb.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_backward_k1_is_identity_on_values():
    q, k, v, rpb, dout = case(2, 2, 5, 7, 8, 1, seed=3)
    dq, dk, dv, drpb = oracle.backward(q, k, v, rpb, dout, 1)
    np.testing.assert_array_equal(dv, dout)
    assert not dq.any() and not dk.any() and not drpb.any()


def test_backward_constant_values():
    q, k, v, rpb, dout = case(1, 2, 9, 8, 4, 5, seed=4)
    v[:] = 1.25
    dq, dk, dv, drpb = oracle.backward(q, k, v, rpb, dout, 5)
    np.testing.assert_allclose(dq, 0, atol=1e-12)
    np.testing.assert_allclose(dk, 0, atol=1e-12)
    np.testing.assert_allclose(drpb, 0, atol=1e-12)
    # dv(r, t) = sum over the queries whose window holds (r, t) of P * dout
    _, _, w = oracle.forward_points(q, k, v, rpb, 5,
                                    [(b, h, i, j) for b in range(1) for h in range(2) for i in range(9)
                                     for j in range(8)])
    want = np.zeros_like(v)
    t = 0
    for h in range(2):
        for i in range(9):
            for j in range(8):
                si, sj = brute_window_start(i, 9, 5), brute_window_start(j, 8, 5)
                for a in range(5):
                    for c in range(5):
                        want[0, h, si + a, sj + c] += w[t, a * 5 + c] * dout[0, h, i, j]
                t += 1
    np.testing.assert_allclose(dv, want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("ks", [3, 5, 7])
def test_backward_bias_gradient_of_each_head_sums_to_zero(ks):
    q, k, v, rpb, dout = case(2, 3, 12, 10, 8, ks, seed=ks)
    drpb = oracle.backward(q, k, v, rpb, dout, ks)[3]
    assert np.abs(drpb).max() > 1e-3  # not trivially zero
    np.testing.assert_allclose(drpb.reshape(3, -1).sum(axis=1), 0, atol=1e-10)
