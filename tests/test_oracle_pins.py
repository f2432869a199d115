"""Pins of the fp64 oracle to what the pages and the mathematics fix.

Every check here compares the oracle with something other than itself:
the border drawing of the pages (a golden fixture), a brute-force window
definition, dense masked self-attention through torch fp64 matmul/softmax,
closed forms (k = 1, box filter, 2-D correlation) and invariants
(translation equivariance, normalisation).  A plausible slip anywhere in the
oracle -- dropped bias, bias not divided by sqrt(d), rows and columns
swapped, a wrong clamp, q and k swapped, a missing max subtraction -- fails
at least one of them (tests/test_oracle_mutations.py plants each one).
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from tests.conftest import read_golden
from vision_sliding_window_b200.inputs import WORKLOADS, make_inputs


def brute_window_start(i, L, ks):
    """Among all ks-wide windows inside [0, L) that contain position i, the
    one whose centre is nearest to i (Neighborhood Attention Transformer,
    Sec. 3.1: the k nearest neighbours; Sec. 1: every pixel keeps the same
    span).  Found by exhaustive search, not by the clamp formula."""
    best = None
    for s in range(0, L - ks + 1):
        if s <= i < s + ks:
            dist = abs(s + (ks - 1) / 2 - i)
            if best is None or dist < best[0]:
                best = (dist, s)
    return best[1]


def dense_masked_attention(q, k, v, rpb, ks):
    """Full self-attention over all H*W keys (Eq. (1) with the bias of Eq. (2))
    restricted by an additive -inf mask to each query's neighbourhood, with
    the bias gathered from the table by displacement.  torch fp64."""
    q, k, v = (torch.as_tensor(np.asarray(x), dtype=torch.float64) for x in (q, k, v))
    B, heads, H, W, d = q.shape
    sr = torch.tensor([brute_window_start(i, H, ks) for i in range(H)])
    sc = torch.tensor([brute_window_start(j, W, ks) for j in range(W)])
    rr, tt = torch.arange(H), torch.arange(W)
    in_r = (rr[None, :] >= sr[:, None]) & (rr[None, :] < sr[:, None] + ks)  # [i, r]
    in_c = (tt[None, :] >= sc[:, None]) & (tt[None, :] < sc[:, None] + ks)  # [j, t]
    mask = in_r[:, None, :, None] & in_c[None, :, None, :]  # [i, j, r, t]
    dr = (rr[None, :] - rr[:, None] + ks - 1).clamp(0, 2 * ks - 2)  # [i, r]
    dc = (tt[None, :] - tt[:, None] + ks - 1).clamp(0, 2 * ks - 2)  # [j, t]
    logits = torch.einsum("bhijx,bhrtx->bhijrt", q, k)
    if rpb is not None:
        tab = torch.as_tensor(np.asarray(rpb), dtype=torch.float64)
        bias = tab[:, dr[:, None, :, None], dc[None, :, None, :]]  # [h, i, j, r, t]
        logits = logits + bias[None]
    logits = logits.masked_fill(~mask, float("-inf")).reshape(B, heads, H, W, H * W)
    p = torch.softmax(logits / math.sqrt(d), dim=-1)
    out = torch.einsum("bhijn,bhnx->bhijx", p, v.reshape(B, heads, H * W, d))
    return out.numpy(), p.numpy()


def f64(*ts):
    return [None if t is None else t.double().numpy() for t in ts]


# ---------------------------------------------------------------- border rule

def test_border_figure_window_starts():
    meta, rows = read_golden("na_border_figure_k3_L5.txt")
    ks, L = meta["ks"], meta["length"]
    for pos, na_start, sasa_start in rows:
        assert oracle.window_start(pos, L, ks) == na_start
        assert brute_window_start(pos, L, ks) == na_start
        # the SASA window is the centred one: it differs from NA exactly at the borders
        assert (sasa_start == na_start) == (pos - ks // 2 == na_start)


def test_border_figure_through_the_operator():
    """q = 0 and no bias make every weight 1/k^2; with one-hot values the
    output spells out each query's window, which must match the drawing."""
    meta, rows = read_golden("na_border_figure_k3_L5.txt")
    ks, L = meta["ks"], meta["length"]
    H = W = L
    d = H * W
    q = np.zeros((1, 1, H, W, d))
    v = np.eye(d).reshape(1, 1, H, W, d)
    out = oracle.forward(q, q, v, None, ks) * ks * ks
    starts = {pos: s for pos, s, _ in rows}
    for i in range(H):
        for j in range(W):
            want = np.zeros((H, W))
            want[starts[i]:starts[i] + ks, starts[j]:starts[j] + ks] = 1.0
            np.testing.assert_allclose(out[0, 0, i, j].reshape(H, W), want, atol=1e-12)


@pytest.mark.parametrize("L", range(1, 14))
def test_window_rule_matches_nearest_window(L):
    for ks in range(1, L + 1, 2):
        for i in range(L):
            assert oracle.window_start(i, L, ks) == brute_window_start(i, L, ks)


def test_corner_queries_keep_full_window():
    # Sec. 1 / App. C: the corner pixel sees a full ks x ks window that is not centred on it
    H, W, ks = 9, 11, 5
    assert oracle.window_start(0, H, ks) == 0 and oracle.window_start(H - 1, H, ks) == H - ks
    assert oracle.window_start(0, W, ks) == 0 and oracle.window_start(W - 1, W, ks) == W - ks
    # all queries within ks//2 of the top edge share the same rows ("repeated windows")
    assert {oracle.window_start(i, H, ks) for i in range(ks // 2 + 1)} == {0}


# ----------------------------------------------------- dense formulation / SA

@pytest.mark.parametrize("B,heads,H,W,d,ks", [
    (1, 1, 5, 5, 4, 3), (2, 3, 6, 9, 8, 3), (1, 2, 7, 5, 16, 5), (2, 1, 9, 8, 4, 7), (1, 1, 4, 6, 3, 1),
])
def test_oracle_equals_dense_masked_attention(B, heads, H, W, d, ks):
    q, k, v, rpb = f64(*make_inputs(B, heads, H, W, d, ks, "f32", seed=11, rpb_std=0.5))
    want, p = dense_masked_attention(q, k, v, rpb, ks)
    got = oracle.forward(q, k, v, rpb, ks)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
    # the unfused chain (Eq. 2, softmax, Eqs. 3-4) gives the same
    attn = oracle.qk_rpb(q, k, rpb, ks)
    probs = oracle.softmax(attn, 1.0 / math.sqrt(d))
    np.testing.assert_allclose(oracle.av(probs, v, ks), want, rtol=0, atol=1e-12)
    # the softmax weights of each window are the non-zero entries of the dense rows
    dense_rows = p.reshape(B, heads, H, W, H * W)
    np.testing.assert_allclose(np.sort(probs, -1), np.sort(dense_rows, -1)[..., -ks * ks:], atol=1e-12)
    np.testing.assert_allclose(probs.sum(-1), 1.0, atol=1e-12)


def test_k_equals_map_is_full_self_attention():
    """NA with the largest neighbourhood is SA (Sec. 3.1 last paragraph): no mask at
    all, the full bias matrix B_full[p, p'] = table[dr + k - 1, dc + k - 1]."""
    w = WORKLOADS["tiny_sa"]
    q, k, v, rpb = f64(*make_inputs(w.B, w.heads, w.H, w.W, w.d, w.ks, "f32", seed=0, rpb_std=0.5))
    n = w.H * w.W
    Q, K, V = (torch.tensor(x.reshape(n, w.d)) for x in (q, k, v))
    pos = torch.tensor([(i, j) for i in range(w.H) for j in range(w.W)])
    disp = pos[None, :, :] - pos[:, None, :] + (w.ks - 1)  # key - query
    bfull = torch.tensor(rpb[0])[disp[..., 0], disp[..., 1]]
    sa = torch.softmax((Q @ K.T + bfull) / math.sqrt(w.d), dim=-1) @ V
    got = oracle.forward(q, k, v, rpb, w.ks)
    np.testing.assert_allclose(got.reshape(n, w.d), sa.numpy(), atol=1e-12)


# ------------------------------------------------------------- closed forms

def test_k1_is_identity_on_values():
    q, k, v, rpb = f64(*make_inputs(2, 2, 5, 6, 8, 1, "f32", seed=3, rpb_std=1.0))
    np.testing.assert_array_equal(oracle.forward(q, k, v, rpb, 1), v)
    attn = oracle.qk_rpb(q, k, rpb, 1)
    want = (q * k).sum(-1) + rpb[None, :, None, None, 0, 0]
    np.testing.assert_allclose(attn[..., 0], want, atol=1e-12)


@pytest.mark.parametrize("H,W,ks", [(9, 9, 3), (8, 11, 5), (7, 7, 7), (12, 5, 5)])
def test_zero_query_no_bias_is_box_filter(H, W, ks):
    """q = 0 and no bias: every weight is 1/k^2, so the output is the mean of v
    over the clamped window, computed here with an integral image."""
    _, _, v, _ = f64(*make_inputs(1, 2, H, W, 4, ks, "f32", seed=5))
    q = np.zeros_like(v)
    got = oracle.forward(q, q, v, None, ks)
    S = np.zeros((1, 2, H + 1, W + 1, 4))
    S[:, :, 1:, 1:] = v.cumsum(2).cumsum(3)
    for i in range(H):
        r0 = brute_window_start(i, H, ks)
        for j in range(W):
            c0 = brute_window_start(j, W, ks)
            tot = S[:, :, r0 + ks, c0 + ks] - S[:, :, r0, c0 + ks] - S[:, :, r0 + ks, c0] + S[:, :, r0, c0]
            np.testing.assert_allclose(got[:, :, i, j], tot / ks**2, atol=1e-12)


@pytest.mark.parametrize("d", [4, 32])
def test_zero_query_bias_is_correlation_kernel(d):
    """q = 0 with a bias table: an interior query's weights are
    softmax(centre block of the table / sqrt(d)) -- the bias is divided by sqrt(d)
    with the dot product (Eq. 4) and indexed by displacement (key - query) --
    so interior outputs are a 2-D correlation of v with that fixed kernel."""
    H, W, ks, heads = 13, 12, 5, 2
    _, _, v, rpb = f64(*make_inputs(1, heads, H, W, d, ks, "f32", seed=7, rpb_std=1.5))
    q = np.zeros_like(v)
    got = oracle.forward(q, q, v, rpb, ks)
    c = ks // 2
    for h in range(heads):
        kern = torch.softmax(torch.tensor(rpb[h, c:c + ks, c:c + ks]).reshape(-1) / math.sqrt(d), 0).reshape(ks, ks)
        img = torch.tensor(v[0, h]).permute(2, 0, 1)[None]  # [1, d, H, W]
        corr = F.conv2d(img, kern.expand(d, 1, ks, ks).contiguous(), groups=d)[0].permute(1, 2, 0).numpy()
        np.testing.assert_allclose(got[0, h, c:H - c, c:W - c], corr, atol=1e-12)


def test_bias_displacement_convention():
    """Reading of B(i, rho_j(i)): table[key_row - query_row + k - 1][key_col - query_col + k - 1].
    A single large entry at displacement (+1, 0) makes an interior query copy the
    value one row below it.  (Which sign the pages mean is not fixed by them.)"""
    H, W, ks, d = 9, 9, 5, 4
    _, _, v, _ = f64(*make_inputs(1, 1, H, W, d, ks, "f32", seed=9))
    q = np.zeros_like(v)
    rpb = np.zeros((1, 2 * ks - 1, 2 * ks - 1))
    rpb[0, ks - 1 + 1, ks - 1] = 400.0
    got = oracle.forward(q, q, v, rpb, ks)
    np.testing.assert_allclose(got[0, 0, 4, 4], v[0, 0, 5, 4], atol=1e-12)


def test_translation_equivariance_away_from_borders():
    """App. C: NA commutes with translation except where windows are clamped."""
    ks, d, Hc = 5, 8, 12
    q, k, v, rpb = f64(*make_inputs(1, 2, 20, 20, d, ks, "f32", seed=13, rpb_std=0.5))
    dy, dx = 3, 5

    def crop(t, y, x):
        return np.ascontiguousarray(t[:, :, y:y + Hc, x:x + Hc])

    a = oracle.forward(crop(q, 0, 0), crop(k, 0, 0), crop(v, 0, 0), rpb, ks)
    b = oracle.forward(crop(q, dy, dx), crop(k, dy, dx), crop(v, dy, dx), rpb, ks)
    c = ks // 2
    checked = 0
    for i in range(dy + c, Hc - c):
        for j in range(dx + c, Hc - c):
            np.testing.assert_allclose(a[:, :, i, j], b[:, :, i - dy, j - dx], atol=1e-12)
            checked += 1
    assert checked > 10
    # ... and it is relaxed at the corner: pixel (dy, dx) is a border query of crop b
    assert not np.allclose(a[:, :, dy, dx], b[:, :, 0, 0])


# -------------------------------------------------------------- invariants

def test_constant_values_give_constant_output():
    q, k, _, rpb = f64(*make_inputs(2, 2, 8, 7, 16, 5, "f32", seed=17, rpb_std=0.5))
    v = np.full_like(q, 2.5)
    np.testing.assert_allclose(oracle.forward(q, k, v, rpb, 5), 2.5, atol=1e-12)


def test_large_logits_stay_finite():
    """The max is subtracted before exp: logits of size 1e4 give a one-hot softmax."""
    q, k, v, _ = f64(*make_inputs(1, 1, 6, 6, 8, 3, "f32", seed=19))
    q = q * 1e4
    out = oracle.forward(q, k, v, None, 3)
    assert np.isfinite(out).all()
    attn = oracle.qk_rpb(q, k, None, 3)
    for i in range(6):
        for j in range(6):
            n = int(np.argmax(attn[0, 0, i, j]))
            r = brute_window_start(i, 6, 3) + n // 3
            t = brute_window_start(j, 6, 3) + n % 3
            np.testing.assert_allclose(out[0, 0, i, j], v[0, 0, r, t], atol=1e-9)


def test_av_with_one_hot_weights_gathers_neighbour():
    H, W, ks, d = 7, 8, 3, 4
    _, _, v, _ = f64(*make_inputs(1, 1, H, W, d, ks, "f32", seed=23))
    rng = np.random.default_rng(0)
    n_sel = rng.integers(0, ks * ks, size=(1, 1, H, W))
    attn = np.zeros((1, 1, H, W, ks * ks))
    np.put_along_axis(attn, n_sel[..., None], 1.0, axis=-1)
    out = oracle.av(attn, v, ks)
    for i in range(H):
        for j in range(W):
            n = n_sel[0, 0, i, j]
            r = brute_window_start(i, H, ks) + n // ks
            t = brute_window_start(j, W, ks) + n % ks
            np.testing.assert_array_equal(out[0, 0, i, j], v[0, 0, r, t])


def test_points_and_rows_agree_with_full_map():
    q, k, v, rpb = f64(*make_inputs(2, 2, 9, 10, 8, 5, "f32", seed=29, rpb_std=0.3))
    full = oracle.forward(q, k, v, rpb, 5)
    pts = [(0, 0, 0, 0), (1, 1, 8, 9), (0, 1, 4, 5), (1, 0, 2, 9)]
    out, logits, w = oracle.forward_points(q, k, v, rpb, 5, pts)
    for t, (b, h, i, j) in enumerate(pts):
        np.testing.assert_allclose(out[t], full[b, h, i, j], atol=1e-13)
    attn = oracle.qk_rpb(q, k, rpb, 5)
    for t, (b, h, i, j) in enumerate(pts):
        np.testing.assert_allclose(logits[t], attn[b, h, i, j], atol=1e-13)
    np.testing.assert_allclose(w.sum(-1), 1.0, atol=1e-13)
    rows = oracle.forward_rows(q, k, v, rpb, 5, 9, 27)
    np.testing.assert_allclose(rows.reshape(-1, 10, 8)[9:27], full.reshape(-1, 10, 8)[9:27], atol=1e-13)


def test_thread_count_does_not_change_results():
    q, k, v, rpb = f64(*make_inputs(1, 3, 10, 10, 8, 5, "f32", seed=31))
    np.testing.assert_array_equal(oracle.forward(q, k, v, rpb, 5, nthreads=1),
                                  oracle.forward(q, k, v, rpb, 5, nthreads=4))


def test_flop_model_is_na_part_of_complexity():
    """Sec. 3.4 and the Qiita complexity section: computing A costs h*w*d*k^2 and
    applying it costs h*w*d*k^2 multiply-adds per head; at 2 FLOPs per
    multiply-add the benchmark's FLOP count is 4*B*heads*H*W*k^2*d."""
    for w in WORKLOADS.values():
        macs_per_head_map = 2 * w.H * w.W * w.d * w.ks ** 2
        assert w.flops == 2 * macs_per_head_map * w.B * w.heads
