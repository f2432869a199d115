"""The C-ABI library without a GPU: it loads, exports every function that
include/na2d.h declares (and nothing else), and rejects bad arguments on the
host before any CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

from vision_sliding_window_b200 import build, na2d

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "na2d.h")
FAKE = 0x10000  # a 16-byte aligned address nothing ever dereferences: every call below fails first


@pytest.fixture(scope="module")
def lib():
    build.build()
    return na2d.load_library()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return set(re.findall(r"\b(na2?d?_\w+)\s*\(", text)) - {"na_status", "na_dtype"}


def test_header_declares_the_binding_exports():
    assert header_functions() == set(na2d.EXPORTS)


def test_library_exports_exactly_the_header(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", na2d.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    funcs = {line.split()[-1] for line in out.splitlines() if " T " in line}
    ours = {f for f in funcs if f.startswith("na")}
    assert ours == header_functions()
    for name in header_functions():
        assert hasattr(lib, name)


def test_status_strings(lib):
    for code, name in enumerate(["NA_OK", "NA_ERR_INVALID_ARG", "NA_ERR_UNSUPPORTED", "NA_ERR_CUDA",
                                 "NA_ERR_DEVICE_TIMEOUT"]):
        assert na2d.status_str(code) == name


def fwd(lib, q=FAKE, k=FAKE, v=FAKE, rpb=None, out=FAKE, B=1, heads=1, H=8, W=8, d=32, ks=3, dt=na2d.NA_BF16):
    return lib.na2d_forward(q, k, v, rpb, out, B, heads, H, W, d, ks, dt, None)


@pytest.mark.parametrize("kw", [
    dict(ks=4), dict(ks=0), dict(ks=-1), dict(ks=9), dict(H=5, ks=7), dict(W=2, ks=3), dict(ks=65, H=70, W=70),
    dict(d=48), dict(d=8), dict(d=0), dict(H=0), dict(W=-3), dict(B=-1), dict(heads=-2), dict(dt=7),
    dict(q=None), dict(k=None), dict(v=None), dict(out=None),
    dict(q=FAKE + 8), dict(out=FAKE + 2), dict(rpb=FAKE + 4), dict(B=1 << 30, heads=1 << 10, H=1 << 10, W=1 << 10),
])
def test_forward_rejects_bad_arguments(lib, kw):
    assert fwd(lib, **kw) == na2d.NA_ERR_INVALID_ARG


def test_empty_batch_is_a_noop(lib):
    assert fwd(lib, B=0) == na2d.NA_OK
    assert fwd(lib, heads=0) == na2d.NA_OK
    assert lib.na2d_qk_rpb(FAKE, FAKE, None, FAKE, 0, 2, 8, 8, 32, 3, na2d.NA_F16, None) == na2d.NA_OK
    assert lib.na2d_av(FAKE, FAKE, FAKE, 3, 0, 8, 8, 32, 3, na2d.NA_F16, None) == na2d.NA_OK
    assert lib.na2d_softmax(FAKE, 0, 1, 8, 8, 3, ctypes.c_float(0.5), None) == na2d.NA_OK


def test_unfused_calls_reject_bad_arguments(lib):
    bad = na2d.NA_ERR_INVALID_ARG
    assert lib.na2d_qk_rpb(None, FAKE, None, FAKE, 1, 1, 8, 8, 32, 3, na2d.NA_F16, None) == bad
    assert lib.na2d_qk_rpb(FAKE, FAKE, None, FAKE + 4, 1, 1, 8, 8, 32, 3, na2d.NA_F16, None) == bad
    assert lib.na2d_qk_rpb(FAKE, FAKE, None, FAKE, 1, 1, 8, 8, 32, 2, na2d.NA_F16, None) == bad
    assert lib.na2d_av(FAKE, FAKE, None, 1, 1, 8, 8, 32, 3, na2d.NA_F16, None) == bad
    assert lib.na2d_av(FAKE, FAKE, FAKE, 1, 1, 8, 8, 24, 3, na2d.NA_F16, None) == bad
    assert lib.na2d_softmax(None, 1, 1, 8, 8, 3, ctypes.c_float(0.5), None) == bad
    assert lib.na2d_softmax(FAKE, 1, 1, 8, 8, 3, ctypes.c_float(float("inf")), None) == bad
    assert lib.na2d_softmax(FAKE, 1, 1, 2, 8, 3, ctypes.c_float(0.5), None) == bad


def test_host_entry_point_checks_workspace(lib):
    need = lib.na2d_forward_host_workspace_bytes(2, 2, 16, 16, 32, 7, na2d.NA_BF16)
    tensor = 2 * 2 * 16 * 16 * 32 * 2
    assert need >= 4 * tensor + 2 * 13 * 13 * 2 and need % 256 == 0
    assert lib.na2d_forward_host_workspace_bytes(2, 2, 16, 16, 32, 8, na2d.NA_BF16) == 0
    args = (FAKE, FAKE, FAKE, None, FAKE)
    assert lib.na2d_forward_host(*args, FAKE, need - 1, 2, 2, 16, 16, 32, 7, na2d.NA_BF16, None) == na2d.NA_ERR_INVALID_ARG
    assert lib.na2d_forward_host(*args, FAKE + 16, need, 2, 2, 16, 16, 32, 7, na2d.NA_BF16, None) == na2d.NA_ERR_INVALID_ARG
    assert lib.na2d_forward_host(*args, None, need, 2, 2, 16, 16, 32, 7, na2d.NA_BF16, None) == na2d.NA_ERR_INVALID_ARG


def test_forward_kernel_selection(lib):
    # float32 always runs the SIMT kernel; rejected shapes report the negated status
    assert lib.na2d_forward_kernel(1, 1, 14, 14, 32, 7, na2d.NA_F32) == 0
    assert lib.na2d_forward_kernel(1, 1, 14, 14, 32, 8, na2d.NA_F32) == -na2d.NA_ERR_INVALID_ARG
    for dt in (na2d.NA_F16, na2d.NA_BF16):
        assert lib.na2d_forward_kernel(32, 2, 56, 56, 32, 7, dt) in (0, 1)


def test_every_benchmarked_16_bit_workload_runs_on_the_tensor_core_kernel(lib):
    from vision_sliding_window_b200.inputs import WORKLOADS

    dts = {"f16": na2d.NA_F16, "bf16": na2d.NA_BF16}
    for w in WORKLOADS.values():
        if w.dtype in dts:
            assert lib.na2d_forward_kernel(w.B, w.heads, w.H, w.W, w.d, w.ks, dts[w.dtype]) == 1, w.name
    # every odd k from 3 to 13 at d = 32 and d = 64
    for d in (32, 64):
        for ks in range(3, 14, 2):
            assert lib.na2d_forward_kernel(2, 2, 40, 40, d, ks, na2d.NA_BF16) == 1, (d, ks)


def test_timeout_probe_rejects_bad_limits(lib):
    assert lib.na2d_debug_timeout_probe(0, None) == na2d.NA_ERR_INVALID_ARG
    assert lib.na2d_debug_timeout_probe(2_000_000, None) == na2d.NA_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(tmp_path):
    saved = na2d._lib
    na2d._lib = None
    try:
        with pytest.raises(RuntimeError, match="missing"):
            na2d.load_library(str(tmp_path / "nope.so"))
    finally:
        na2d._lib = saved


def bwd(lib, q=FAKE, k=FAKE, v=FAKE, rpb=None, dout=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, drpb=FAKE, ws=FAKE,
        ws_bytes=1 << 30, B=1, heads=1, H=8, W=8, d=32, ks=3, dt=na2d.NA_BF16):
    return lib.na2d_backward(q, k, v, rpb, dout, dq, dk, dv, drpb, ws, ws_bytes, B, heads, H, W, d, ks, dt, None)


@pytest.mark.parametrize("kw", [
    dict(ks=4), dict(ks=11), dict(d=48), dict(H=0), dict(dt=5), dict(q=None), dict(dout=None), dict(dq=None),
    dict(dk=None), dict(dv=None), dict(ws=None), dict(q=FAKE + 8), dict(dv=FAKE + 2), dict(drpb=FAKE + 4),
    dict(rpb=FAKE + 4), dict(ws=FAKE + 8), dict(ws_bytes=16 * 64 - 1),
])
def test_backward_rejects_bad_arguments(lib, kw):
    assert bwd(lib, **kw) == na2d.NA_ERR_INVALID_ARG


def test_backward_workspace_and_empty_batch(lib):
    # two float64 per query
    assert lib.na2d_backward_workspace_bytes(2, 3, 10, 12, 32, 5, na2d.NA_F16) == 16 * 2 * 3 * 10 * 12
    assert lib.na2d_backward_workspace_bytes(2, 3, 10, 12, 32, 4, na2d.NA_F16) == 0
    assert bwd(lib, B=0, q=None, dq=None, ws=None) == na2d.NA_OK


def test_sasa_arguments(lib):
    # any odd k, even one larger than the map; workspace: padded q, k, v and output
    need = lib.na2d_sasa_workspace_bytes(1, 1, 5, 6, 32, 7, na2d.NA_BF16)
    assert need == 4 * ((1 * 1 * 11 * 12 * 32 * 2 + 255) // 256 * 256)
    assert lib.na2d_sasa_workspace_bytes(1, 1, 5, 6, 32, 8, na2d.NA_BF16) == 0
    args = (FAKE, FAKE, FAKE, None, FAKE)
    assert lib.na2d_sasa_forward(*args, FAKE, need - 1, 1, 1, 5, 6, 32, 7, na2d.NA_BF16, None) == na2d.NA_ERR_INVALID_ARG
    assert lib.na2d_sasa_forward(*args, FAKE + 16, need, 1, 1, 5, 6, 32, 7, na2d.NA_BF16, None) == na2d.NA_ERR_INVALID_ARG
    assert lib.na2d_sasa_forward(None, FAKE, FAKE, None, FAKE, FAKE, need, 1, 1, 5, 6, 32, 7, na2d.NA_BF16,
                                 None) == na2d.NA_ERR_INVALID_ARG
    assert lib.na2d_sasa_forward(*args, None, 0, 0, 1, 5, 6, 32, 7, na2d.NA_BF16, None) == na2d.NA_OK


def test_block_arguments(lib):
    need = lib.na2d_block_workspace_bytes(2, 8, 8, 2, 32, 3, na2d.NA_BF16)
    assert need > 2 * 8 * 8 * 64 * (3 * 4 + 5 * 2 + 4)
    assert lib.na2d_block_workspace_bytes(2, 8, 8, 2, 48, 3, na2d.NA_BF16) == 0
    a = (FAKE, FAKE, None, FAKE, None, None, FAKE)
    assert lib.na2d_block_forward(*a, FAKE, need - 1, 2, 8, 8, 2, 32, 3, na2d.NA_BF16, None) == na2d.NA_ERR_INVALID_ARG
    assert lib.na2d_block_forward(*a, FAKE + 16, need, 2, 8, 8, 2, 32, 3, na2d.NA_BF16, None) == na2d.NA_ERR_INVALID_ARG
    assert lib.na2d_block_forward(None, FAKE, None, FAKE, None, None, FAKE, FAKE, need, 2, 8, 8, 2, 32, 3,
                                  na2d.NA_BF16, None) == na2d.NA_ERR_INVALID_ARG
    assert lib.na2d_block_forward(*a, None, 0, 0, 8, 8, 2, 32, 3, na2d.NA_BF16, None) == na2d.NA_OK


@pytest.mark.parametrize("kw", [dict(k2=4), dict(dil1=0), dict(L2=10, dil2=4, k2=3), dict(d=24), dict(q=None),
                                dict(out=FAKE + 8), dict(L0=0)])
def test_nd_rejects_bad_arguments(lib, kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, rpb=None, out=FAKE, B=1, heads=1, L0=1, L1=9, L2=12, d=32, k0=1, k1=3, k2=5,
             dil0=1, dil1=2, dil2=2)
    a.update(kw)
    assert lib.na_forward_nd(*a.values(), na2d.NA_BF16, None) == na2d.NA_ERR_INVALID_ARG
