"""Parity of the CUDA path (through the C ABI) with the fp64 oracle on the
same seeded inputs.

Tolerances: float32 -- |gpu - oracle| <= 1e-6 + 1e-5 |oracle| elementwise;
fp16 / bf16 with float32 accumulation -- max |gpu - oracle| <= 2e-2, for the
output of na2d_forward / na2d_av and for the float32 logits of na2d_qk_rpb.
Small maps are compared in full; the full-size workloads are compared at
sampled query points (corners, edge midpoints and random points, each
computed by the oracle one by one) and checked for finiteness everywhere.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from vision_sliding_window_b200 import build, na2d
from vision_sliding_window_b200.inputs import DTYPES, WORKLOADS, make_inputs, sample_points, workload_inputs

pytestmark = pytest.mark.gpu

MAX_ABS_16 = 2e-2


@pytest.fixture(scope="module", autouse=True)
def lib():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    build.build()
    return na2d.load_library()


def to_dev(*ts):
    return [None if t is None else t.cuda() for t in ts]


def assert_close(got, want, dtype, what=""):
    g = got.detach().double().cpu().numpy() if torch.is_tensor(got) else np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert g.shape == want.shape, (g.shape, want.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    if dtype == "f32":
        np.testing.assert_allclose(g, want, rtol=1e-5, atol=1e-6, err_msg=what)
    else:
        err = np.abs(g - want).max()
        assert err <= MAX_ABS_16, f"{what}: max abs error {err:.3e} > {MAX_ABS_16}"


def run_forward(q, k, v, rpb, ks):
    out = na2d.forward(q, k, v, rpb, ks)
    torch.cuda.synchronize()
    assert na2d.device_status() == na2d.NA_OK
    return out


# ----------------------------------------------------------- the workloads

SMALL = ["tiny", "tiny_sa", "stage3", "stage4", "stage1"]
LARGE = ["hires_k7", "hires_k13"] + [f"sweep_k{k}" for k in (3, 5, 7, 9, 11, 13)]


@pytest.mark.parametrize("name", SMALL)
def test_forward_workload_in_full(name):
    w = WORKLOADS[name]
    q, k, v, rpb = workload_inputs(w)
    out = run_forward(*to_dev(q, k, v, rpb), w.ks)
    assert_close(out, oracle.forward(q, k, v, rpb, w.ks), w.dtype, name)


@pytest.mark.parametrize("name", LARGE)
def test_forward_workload_sampled(name):
    w = WORKLOADS[name]
    q, k, v, rpb = workload_inputs(w)
    out = run_forward(*to_dev(q, k, v, rpb), w.ks)
    assert torch.isfinite(out).all()
    pts = sample_points(w, 3000)
    want, _, _ = oracle.forward_points(q, k, v, rpb, w.ks, pts)
    got = out[pts[:, 0], pts[:, 1], pts[:, 2], pts[:, 3]]
    assert_close(got, want, w.dtype, name)


# Every (dtype, k, d) the tensor-core kernel is built for, compared in full
# with the oracle on maps that give each CTA several work units: 4x2x72x72
# has a last tile row of single tiles (packed two per unit) and 324 units on
# a 148-SM grid; 3x2x75x70 has a ragged last pair row (75 = 4*16 + 11) and a
# ragged last tile column (70 = 8*8 + 6).
TC_BUILDS = [(dt, ks, d) for dt in ("f16", "bf16") for ks in (3, 5, 7, 9, 11, 13) for d in (32, 64)]


@pytest.mark.parametrize("dtype,ks,d", TC_BUILDS)
def test_every_tc_build_in_full(dtype, ks, d):
    for (B, heads, H, W), seed in (((4, 2, 72, 72), 7), ((3, 2, 75, 70), 8)):
        assert na2d.forward_kernel(B, heads, H, W, d, ks, DTYPES[dtype]) == 1
        q, k, v, rpb = make_inputs(B, heads, H, W, d, ks, dtype, seed=seed + ks, rpb_std=0.5)
        out = run_forward(*to_dev(q, k, v, rpb), ks)
        assert_close(out, oracle.forward(q, k, v, rpb, ks), dtype, f"{dtype} k={ks} d={d} {H}x{W}")


@pytest.mark.parametrize("name", LARGE)
def test_forward_workload_first_and_last_map_in_full(name):
    """The first and the last (b, h) map of each large workload, every element."""
    w = WORKLOADS[name]
    q, k, v, rpb = workload_inputs(w)
    out = run_forward(*to_dev(q, k, v, rpb), w.ks).cpu()
    maps = w.B * w.heads
    for m in (0, maps - 1):
        want = oracle.forward_rows(q, k, v, rpb, w.ks, m * w.H, (m + 1) * w.H)
        b, h = divmod(m, w.heads)
        assert_close(out[b, h], want[b, h], w.dtype, f"{name} map {m}")


@pytest.mark.parametrize("dtype,scale", [("bf16", 4.0), ("f16", 4.0), ("bf16", 8.0)])
def test_wide_logit_spread_in_full(dtype, scale):
    """q scaled up so that the scaled logits A/sqrt(d) span tens: the regime
    where a 16-bit exponent argument or a loose shift would cost accuracy."""
    q, k, v, rpb = make_inputs(2, 2, 40, 36, 32, 7, dtype, seed=61, rpb_std=0.5)
    q = (q.float() * scale).to(q.dtype)
    out = run_forward(*to_dev(q, k, v, rpb), 7)
    assert_close(out, oracle.forward(q, k, v, rpb, 7), dtype, f"q x {scale}")


def test_k_equals_map_matches_dense_self_attention_on_gpu():
    """Stage-4 (H = W = k = 7): the output is plain self-attention with the full bias."""
    w = WORKLOADS["stage4"]
    q, k, v, rpb = workload_inputs(w)
    out = run_forward(*to_dev(q, k, v, rpb), w.ks)
    n = w.H * w.W
    Q, K, V = (t.double().reshape(w.B, w.heads, n, w.d) for t in (q, k, v))
    pos = torch.tensor([(i, j) for i in range(w.H) for j in range(w.W)])
    disp = pos[None, :, :] - pos[:, None, :] + (w.ks - 1)
    bfull = rpb.double()[:, disp[..., 0], disp[..., 1]]  # [heads, n, n]
    sa = torch.softmax((Q @ K.transpose(-1, -2) + bfull[None]) / math.sqrt(w.d), -1) @ V
    assert_close(out.reshape(w.B, w.heads, n, w.d), sa.numpy(), w.dtype, "stage4 vs SA")


# -------------------------------------------------------- unfused chain

CHAIN = [("tiny", None), ("stage1", 2000), ("hires_k13", 1500), ("sweep_k5", 1500)]


@pytest.mark.parametrize("name,npts", CHAIN)
def test_unfused_chain(name, npts):
    w = WORKLOADS[name]
    q, k, v, rpb = workload_inputs(w)
    dq, dk, dv, drpb = to_dev(q, k, v, rpb)
    attn = na2d.qk_rpb(dq, dk, drpb, w.ks)
    logits = attn.clone()
    na2d.softmax_(attn, w.ks, 1.0 / math.sqrt(w.d))
    out = na2d.av(attn, dv, w.ks)
    torch.cuda.synchronize()
    if npts is None:
        want_logits = oracle.qk_rpb(q, k, rpb, w.ks)
        assert_close(logits, want_logits, w.dtype, "qk_rpb")
        assert_close(attn, oracle.softmax(want_logits, 1 / math.sqrt(w.d)), "f32", "softmax")
        assert_close(out, oracle.forward(q, k, v, rpb, w.ks), w.dtype, "chain")
        return
    pts = sample_points(w, npts)
    want_out, want_logits, want_w = oracle.forward_points(q, k, v, rpb, w.ks, pts)
    sel = (pts[:, 0], pts[:, 1], pts[:, 2], pts[:, 3])
    assert_close(logits[sel], want_logits, w.dtype, "qk_rpb")
    np.testing.assert_allclose(attn[sel].double().cpu().numpy(), want_w, atol=2e-3)
    assert_close(out[sel], want_out, w.dtype, "chain")


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_softmax_and_av_on_oracle_inputs(dtype):
    """na2d_softmax and na2d_av fed the oracle's own logits / weights."""
    q, k, v, rpb = make_inputs(2, 3, 11, 13, 32, 5, dtype, seed=41)
    logits = oracle.qk_rpb(q, k, rpb, 5)
    dl = torch.tensor(logits, dtype=torch.float32, device="cuda")
    na2d.softmax_(dl, 5, 1 / math.sqrt(32))
    want_w = oracle.softmax(logits.astype(np.float32), 1 / math.sqrt(32))
    np.testing.assert_allclose(dl.double().cpu().numpy(), want_w, rtol=1e-5, atol=1e-7)
    w32 = oracle.softmax(logits, 1 / math.sqrt(32)).astype(np.float32)
    out = na2d.av(torch.tensor(w32, device="cuda"), v.cuda(), 5)
    assert_close(out, oracle.av(w32, v, 5), dtype, "av")


# ------------------------------------------------------------ edge shapes

EDGE = [
    # B, heads, H, W, d, ks, dtype, rpb
    (1, 1, 1, 1, 32, 1, "bf16", True),
    (2, 1, 3, 5, 16, 3, "f16", True),
    (1, 2, 7, 7, 64, 7, "bf16", False),
    (1, 1, 13, 13, 32, 13, "f16", True),
    (1, 1, 14, 13, 32, 13, "bf16", True),
    (3, 2, 57, 9, 32, 7, "bf16", True),
    (1, 3, 9, 57, 32, 9, "f16", True),
    (2, 2, 17, 23, 128, 5, "bf16", True),
    (1, 1, 8, 8, 128, 3, "f32", True),
    (2, 3, 19, 21, 16, 11, "f32", True),
    (1, 2, 33, 31, 64, 1, "f16", True),
    (1, 1, 40, 40, 32, 5, "f32", False),
    (2, 1, 24, 25, 64, 9, "f16", False),
    (1, 1, 129, 130, 32, 13, "bf16", True),
    (1, 1, 16, 16, 32, 15, "bf16", True),
]


@pytest.mark.parametrize("B,heads,H,W,d,ks,dtype,with_rpb", EDGE)
def test_edge_shapes(B, heads, H, W, d, ks, dtype, with_rpb):
    q, k, v, rpb = make_inputs(B, heads, H, W, d, ks, dtype, seed=B * 1000 + H * 10 + ks,
                               rpb_std=0.5, with_rpb=with_rpb)
    out = run_forward(*to_dev(q, k, v, rpb), ks)
    assert_close(out, oracle.forward(q, k, v, rpb, ks), dtype, "forward")
    attn = na2d.qk_rpb(*to_dev(q, k, rpb), ks)
    assert_close(attn, oracle.qk_rpb(q, k, rpb, ks), dtype, "qk_rpb")


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
def test_k1_returns_values(dtype):
    q, k, v, rpb = make_inputs(2, 2, 9, 10, 32, 1, dtype, seed=3, rpb_std=1.0)
    out = run_forward(*to_dev(q, k, v, rpb), 1)
    assert torch.equal(out.cpu(), v)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_constant_values(dtype):
    q, k, _, rpb = make_inputs(2, 2, 30, 20, 32, 7, dtype, seed=5)
    v = torch.full_like(q, 1.5)
    out = run_forward(*to_dev(q, k, v, rpb), 7)
    assert (out.float() - 1.5).abs().max().item() <= 1e-2


def test_large_logits_stay_finite():
    q, k, v, rpb = make_inputs(1, 2, 20, 20, 32, 5, "bf16", seed=8)
    q = (q.float() * 30).to(torch.bfloat16)
    out = run_forward(*to_dev(q, k, v, rpb), 5)
    assert torch.isfinite(out).all()
    assert_close(out, oracle.forward(q, k, v, rpb, 5), "bf16", "large logits")


# ---------------------------------------- outputs written exactly, in place

def guarded(shape, dtype, pad=4096):
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * pad,), float("nan"), dtype=dtype, device="cuda")
    return buf, buf[pad:pad + n].view(shape)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_outputs_written_exactly_once_in_bounds(dtype):
    shp = (2, 2, 23, 29, 32)
    q, k, v, rpb = make_inputs(*shp, 7, dtype, seed=51)
    dq, dk, dv, drpb = to_dev(q, k, v, rpb)
    buf, out = guarded(shp, DTYPES[dtype])
    na2d.forward(dq, dk, dv, drpb, 7, out=out)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    assert torch.isnan(buf[:4096]).all() and torch.isnan(buf[-4096:]).all()
    abuf, attn = guarded(shp[:4] + (49,), torch.float32)
    na2d.qk_rpb(dq, dk, drpb, 7, attn=attn)
    torch.cuda.synchronize()
    assert torch.isfinite(attn).all()
    assert torch.isnan(abuf[:4096]).all() and torch.isnan(abuf[-4096:]).all()
    obuf, out2 = guarded(shp, DTYPES[dtype])
    na2d.av(na2d.softmax_(attn, 7, 32 ** -0.5), dv, 7, out=out2)
    torch.cuda.synchronize()
    assert torch.isfinite(out2).all()
    assert torch.isnan(obuf[:4096]).all() and torch.isnan(obuf[-4096:]).all()


def test_inputs_are_not_modified_and_runs_are_deterministic():
    w = WORKLOADS["stage1"]
    q, k, v, rpb = to_dev(*workload_inputs(w))
    copies = [t.clone() for t in (q, k, v, rpb)]
    a = run_forward(q, k, v, rpb, w.ks)
    b = run_forward(q, k, v, rpb, w.ks)
    assert torch.equal(a, b)
    for t, c in zip((q, k, v, rpb), copies):
        assert torch.equal(t, c)


def test_empty_batch_leaves_output_untouched():
    q = torch.zeros((0, 2, 8, 8, 32), dtype=torch.bfloat16, device="cuda")
    out = na2d.forward(q, q, q, None, 3)
    torch.cuda.synchronize()
    assert out.shape == q.shape


def test_side_stream():
    w = WORKLOADS["stage3"]
    q, k, v, rpb = workload_inputs(w)
    dq, dk, dv, drpb = to_dev(q, k, v, rpb)
    ref = run_forward(dq, dk, dv, drpb, w.ks)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = na2d.forward(dq, dk, dv, drpb, w.ks)
    s.synchronize()
    assert torch.equal(out, ref)


def test_host_buffer_entry_point_matches_device_call():
    w = WORKLOADS["stage1"]
    q, k, v, rpb = workload_inputs(w)
    ref = run_forward(*to_dev(q, k, v, rpb), w.ks).cpu()
    pin = [t.pin_memory() for t in (q, k, v, rpb)]
    out = torch.empty_like(q).pin_memory()
    ws = torch.empty(na2d.host_workspace_bytes(*w.shape(), w.ks, q.dtype), dtype=torch.uint8, device="cuda")
    na2d.forward_host(*pin, out, w.ks, ws)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


# -------------------------------------------------------------- failure path

def test_bounded_wait_reports_timeout_and_context_survives():
    assert na2d.device_status() == na2d.NA_OK
    assert na2d.debug_timeout_probe(2000) == na2d.NA_OK
    assert na2d.device_status() == na2d.NA_ERR_DEVICE_TIMEOUT
    assert na2d.device_status() == na2d.NA_OK  # cleared by the read
    w = WORKLOADS["tiny"]
    q, k, v, rpb = workload_inputs(w)
    out = run_forward(*to_dev(q, k, v, rpb), w.ks)
    assert_close(out, oracle.forward(q, k, v, rpb, w.ks), w.dtype, "after timeout")
