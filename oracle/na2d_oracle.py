"""ctypes front end of the fp64 C oracle (``na2d_oracle.c``).

Test infrastructure only.  Arrays are numpy; everything is converted to
contiguous float64 before the call, which is exact for fp32, fp16 and bf16
values.  The shared object is compiled with gcc on first use (or by
``build()``), next to the source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "na2d_oracle.c")
_LIB = os.path.join(_HERE, "libna2d_oracle.so")
_lock = threading.Lock()
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_L = ctypes.c_long


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, IEEE arithmetic, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.na2d_oracle_window_start.restype = _L
            lib.na2d_oracle_window_start.argtypes = [_L, _L, _L]
            lib.na2d_oracle_qk_rpb.argtypes = [_D, _D, _D, _D] + [_L] * 6 + [ctypes.c_int]
            lib.na2d_oracle_softmax.argtypes = [_D, _L, _L, ctypes.c_double, ctypes.c_int]
            lib.na2d_oracle_av.argtypes = [_D, _D, _D] + [_L] * 6 + [ctypes.c_int]
            lib.na2d_oracle_forward.argtypes = [_D, _D, _D, _D, _D] + [_L] * 6 + [ctypes.c_int]
            lib.na2d_oracle_forward_rows.argtypes = (
                [_D, _D, _D, _D, _D] + [_L] * 6 + [_L, _L, ctypes.c_int]
            )
            lib.na2d_oracle_forward_points.argtypes = (
                [_D, _D, _D, _D, ctypes.POINTER(ctypes.c_int64), _L, _D, _D, _D]
                + [_L] * 6
                + [ctypes.c_int]
            )
            lib.na2d_oracle_backward.argtypes = [_D] * 9 + [_L] * 6 + [ctypes.c_int]
            lib.na2d_oracle_sasa_forward.argtypes = [_D] * 5 + [_L] * 6 + [ctypes.c_int]
            lib.na2d_oracle_nd_forward.argtypes = [_D] * 5 + [_L] * 12 + [ctypes.c_int]
            lib.na2d_oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


class swapped_library:
    """Context manager that points this module at another compiled copy of the
    oracle (used by the test that plants mistakes in a copy of the source)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        _load()
        self._saved = _lib
        lib = ctypes.CDLL(self.path)
        for fn in ("na2d_oracle_window_start", "na2d_oracle_qk_rpb", "na2d_oracle_softmax",
                   "na2d_oracle_av", "na2d_oracle_forward", "na2d_oracle_forward_rows",
                   "na2d_oracle_forward_points", "na2d_oracle_backward", "na2d_oracle_sasa_forward",
                   "na2d_oracle_nd_forward",
                   "na2d_oracle_max_threads"):
            src, dst = getattr(self._saved, fn), getattr(lib, fn)
            dst.argtypes, dst.restype = src.argtypes, src.restype
        with _lock:
            _lib = lib
        return lib

    def __exit__(self, *exc):
        global _lib
        with _lock:
            _lib = self._saved
        return False


def compile_variant(source_text: str, out_path: str) -> str:
    """Compiles a modified copy of the oracle source to out_path."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(source_text)
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", out_path, src, "-lm"])
    return out_path


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # a torch tensor: go through fp32, exact for 16-bit types
        a = a.detach().cpu()
        if a.dtype not in (_torch_f64(),):
            a = a.float()
        a = a.numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _torch_f64():
    import torch

    return torch.float64


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_D)


def _shape(q, ks):
    B, heads, H, W, d = q.shape
    if ks % 2 != 1 or ks < 1 or ks > H or ks > W:
        raise ValueError(f"kernel size {ks} must be odd and fit the {H}x{W} map")
    return B, heads, H, W, d


def window_start(i: int, L: int, ks: int) -> int:
    return int(_load().na2d_oracle_window_start(i, L, ks))


def max_threads() -> int:
    return int(_load().na2d_oracle_max_threads())


def qk_rpb(q, k, rpb, ks: int, nthreads: int = 0) -> np.ndarray:
    """Unscaled Eq. (2) logits, [B, heads, H, W, ks*ks]."""
    q, k, rpb = _f64(q), _f64(k), _f64(rpb)
    B, heads, H, W, d = _shape(q, ks)
    attn = np.empty((B, heads, H, W, ks * ks), dtype=np.float64)
    _load().na2d_oracle_qk_rpb(_ptr(q), _ptr(k), _ptr(rpb), _ptr(attn), B, heads, H, W, d, ks, nthreads)
    return attn


def softmax(attn, scale: float, nthreads: int = 0) -> np.ndarray:
    """softmax(scale * attn) over the last axis (length ks*ks)."""
    a = np.array(_f64(attn), dtype=np.float64, copy=True)
    kk = a.shape[-1]
    ks = int(round(kk ** 0.5))
    assert ks * ks == kk
    _load().na2d_oracle_softmax(_ptr(a), a.size // kk, ks, float(scale), nthreads)
    return a


def av(attn, v, ks: int, nthreads: int = 0) -> np.ndarray:
    """Eqs. (3)-(4) with given weights: [B, heads, H, W, d]."""
    attn, v = _f64(attn), _f64(v)
    B, heads, H, W, d = _shape(v, ks)
    out = np.empty_like(v)
    _load().na2d_oracle_av(_ptr(attn), _ptr(v), _ptr(out), B, heads, H, W, d, ks, nthreads)
    return out


def forward(q, k, v, rpb, ks: int, nthreads: int = 0) -> np.ndarray:
    """NA_k of Eq. (4) over the whole map: [B, heads, H, W, d]."""
    q, k, v, rpb = _f64(q), _f64(k), _f64(v), _f64(rpb)
    B, heads, H, W, d = _shape(q, ks)
    out = np.empty_like(q)
    _load().na2d_oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(rpb), _ptr(out), B, heads, H, W, d, ks, nthreads)
    return out


def forward_rows(q, k, v, rpb, ks: int, row_begin: int, row_end: int, nthreads: int = 0) -> np.ndarray:
    """NA_k for flattened rows [row_begin, row_end) of (b, h, i); returns the full-shape
    output array with only those rows written (the rest is zero)."""
    q, k, v, rpb = _f64(q), _f64(k), _f64(v), _f64(rpb)
    B, heads, H, W, d = _shape(q, ks)
    out = np.zeros_like(q)
    _load().na2d_oracle_forward_rows(
        _ptr(q), _ptr(k), _ptr(v), _ptr(rpb), _ptr(out), B, heads, H, W, d, ks, row_begin, row_end, nthreads
    )
    return out


def forward_points(q, k, v, rpb, ks: int, points, nthreads: int = 0):
    """NA_k at the listed (b, h, i, j) points.

    Returns (out [n, d], logits [n, ks*ks] unscaled, weights [n, ks*ks])."""
    q, k, v, rpb = _f64(q), _f64(k), _f64(v), _f64(rpb)
    B, heads, H, W, d = _shape(q, ks)
    pts = np.ascontiguousarray(np.asarray(points, dtype=np.int64).reshape(-1, 4))
    n = pts.shape[0]
    out = np.empty((n, d), dtype=np.float64)
    logits = np.empty((n, ks * ks), dtype=np.float64)
    attn = np.empty((n, ks * ks), dtype=np.float64)
    _load().na2d_oracle_forward_points(
        _ptr(q), _ptr(k), _ptr(v), _ptr(rpb),
        pts.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n,
        _ptr(out), _ptr(logits), _ptr(attn), B, heads, H, W, d, ks, nthreads,
    )
    return out, logits, attn


def backward(q, k, v, rpb, dout, ks: int, nthreads: int = 0):
    """Gradients of L = sum(dout * NA_k(q, k, v, rpb)) with respect to q, k,
    v and rpb (the backward of Eqs. (2)-(4)).  Returns (dq, dk, dv, drpb);
    drpb is None when rpb is None."""
    q, k, v, rpb, dout = _f64(q), _f64(k), _f64(v), _f64(rpb), _f64(dout)
    B, heads, H, W, d = _shape(q, ks)
    dq, dk, dv = (np.empty_like(q) for _ in range(3))
    drpb = None if rpb is None else np.empty_like(rpb)
    _load().na2d_oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(rpb), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                 _ptr(drpb), B, heads, H, W, d, ks, nthreads)
    return dq, dk, dv, drpb


def sasa_forward(q, k, v, rpb, ks: int, nthreads: int = 0) -> np.ndarray:
    """SASA: the centred ks x ks window with zero keys and values outside the
    map (NA on a zero-padded input, NAT Sec. 3.2): [B, heads, H, W, d]."""
    q, k, v, rpb = _f64(q), _f64(k), _f64(v), _f64(rpb)
    B, heads, H, W, d = q.shape
    if ks % 2 != 1 or ks < 1:
        raise ValueError(f"kernel size {ks} must be odd")
    out = np.empty_like(q)
    _load().na2d_oracle_sasa_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(rpb), _ptr(out), B, heads, H, W, d, ks,
                                     nthreads)
    return out


def _round_to(a, dtype_name):
    """a rounded to fp16 / bf16 (round-to-nearest-even), back in float64."""
    if dtype_name in (None, "f32"):
        return a
    import torch

    t = {"f16": torch.float16, "bf16": torch.bfloat16}[dtype_name]
    return torch.from_numpy(np.ascontiguousarray(a)).to(t).double().numpy()


def block_forward(x, wqkv, bqkv, wo, bo, rpb, heads: int, ks: int, store=None, nthreads: int = 0):
    """An NA block (NAT App. A.1: linear projections for queries, keys and
    values, NA, a final linear projection; Qiita "計算量": 4hwd^2 + 2hwdk^2):

        qkv = x Wqkv + bqkv          x [B, H, W, C], Wqkv [C, 3C]
        q, k, v = the three C-channel thirds of qkv, each as heads x dh
        o = NA_ks(q, k, v, rpb)      per head
        y = o Wo + bo                o as [B, H, W, heads * dh], Wo [C, C]

    store: None for plain float64, or "f16" / "bf16": q, k, v and o are
    rounded to that type where a 16-bit model stores them, and y at the end.
    Returns y [B, H, W, C]."""
    x, wqkv, wo = (np.asarray(_f64(t)) for t in (x, wqkv, wo))
    bqkv = None if bqkv is None else np.asarray(_f64(bqkv))
    bo = None if bo is None else np.asarray(_f64(bo))
    B, H, W, C = x.shape
    dh = C // heads
    qkv = x.reshape(-1, C) @ wqkv
    if bqkv is not None:
        qkv = qkv + bqkv
    qkv = _round_to(qkv, store).reshape(B, H, W, 3, heads, dh)
    q, k, v = (np.ascontiguousarray(qkv[:, :, :, s].transpose(0, 3, 1, 2, 4)) for s in range(3))
    o = _round_to(forward(q, k, v, rpb, ks, nthreads), store)  # [B, heads, H, W, dh]
    y = o.transpose(0, 2, 3, 1, 4).reshape(-1, C) @ wo
    if bo is not None:
        y = y + bo
    return _round_to(y, store).reshape(B, H, W, C)


def nd_forward(q, k, v, rpb, ks, dilation=None, nthreads: int = 0) -> np.ndarray:
    """NA over the trailing 1, 2 or 3 spatial axes of q [B, heads, *spatial, d]
    with per-axis kernel sizes ks and dilations (the sub-grid reading: a
    query attends within the positions congruent to it mod the dilation, with
    NA's clamped window there).  rpb [heads, *(2k - 1)] or None."""
    q, k, v, rpb = _f64(q), _f64(k), _f64(v), _f64(rpb)
    nsp = q.ndim - 3
    if nsp not in (1, 2, 3):
        raise ValueError("q must be [B, heads, *spatial, d] with 1-3 spatial axes")
    ks = tuple(ks) if hasattr(ks, "__len__") else (ks,) * nsp
    dilation = tuple(dilation) if dilation is not None else (1,) * nsp
    B, heads, d = q.shape[0], q.shape[1], q.shape[-1]
    L = (1,) * (3 - nsp) + tuple(q.shape[2:-1])
    kk = (1,) * (3 - nsp) + ks
    dl = (1,) * (3 - nsp) + dilation
    for La, ka, da in zip(L, kk, dl):
        if ka % 2 != 1 or da < 1 or La // da < ka:
            raise ValueError(f"axis of length {La}: kernel {ka} (odd) and dilation {da} need L // dilation >= kernel")
    if rpb is not None:
        rpb = np.ascontiguousarray(rpb.reshape(heads, 2 * kk[0] - 1, 2 * kk[1] - 1, 2 * kk[2] - 1))
    out = np.empty_like(q)
    _load().na2d_oracle_nd_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(rpb), _ptr(out), B, heads, *L, d, *kk, *dl,
                                   nthreads)
    return out
