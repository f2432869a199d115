"""Python binding of libna2d.so (include/na2d.h), through ctypes.

Argument marshalling only: every step of the operator runs in the
library's CUDA kernels.  PyTorch supplies device memory and the current
stream.  If the shared library is missing the import of this module
succeeds but every call raises -- there is no other implementation.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libna2d.so")

NA_OK, NA_ERR_INVALID_ARG, NA_ERR_UNSUPPORTED, NA_ERR_CUDA, NA_ERR_DEVICE_TIMEOUT = range(5)
NA_F32, NA_F16, NA_BF16 = 0, 1, 2
_DT = {torch.float32: NA_F32, torch.float16: NA_F16, torch.bfloat16: NA_BF16}

# Every exported symbol of include/na2d.h.
EXPORTS = (
    "na2d_qk_rpb", "na2d_softmax", "na2d_av", "na2d_forward",
    "na2d_forward_host_workspace_bytes", "na2d_forward_host", "na2d_forward_host_noalloc", "na2d_forward_kernel",
    "na2d_device_status", "na2d_debug_timeout_probe", "na_status_str",
    "na2d_backward_workspace_bytes", "na2d_backward", "na2d_sasa_workspace_bytes", "na2d_sasa_forward",
    "na2d_block_workspace_bytes", "na2d_block_forward", "na_forward_nd",
)


class NA2DError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_str(status)}")


_lock = threading.Lock()
_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with `python -m vision_sliding_window_b200.build`"
            )
        lib = ctypes.CDLL(path)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        shape = [i] * 6
        lib.na2d_qk_rpb.argtypes = [vp, vp, vp, vp, *shape, i, vp]
        lib.na2d_softmax.argtypes = [vp, i, i, i, i, i, f, vp]
        lib.na2d_av.argtypes = [vp, vp, vp, *shape, i, vp]
        lib.na2d_forward.argtypes = [vp, vp, vp, vp, vp, *shape, i, vp]
        lib.na2d_forward_host_workspace_bytes.argtypes = [*shape, i]
        lib.na2d_forward_host_workspace_bytes.restype = sz
        lib.na2d_forward_host.argtypes = [vp, vp, vp, vp, vp, vp, sz, *shape, i, vp]
        lib.na2d_forward_host_noalloc.argtypes = [vp, vp, vp, vp, vp, *shape, i, vp]
        lib.na2d_forward_kernel.argtypes = [*shape, i]
        lib.na2d_backward_workspace_bytes.argtypes = [*shape, i]
        lib.na2d_backward_workspace_bytes.restype = sz
        lib.na2d_backward.argtypes = [vp] * 10 + [sz, *shape, i, vp]
        lib.na2d_sasa_workspace_bytes.argtypes = [*shape, i]
        lib.na2d_sasa_workspace_bytes.restype = sz
        lib.na2d_sasa_forward.argtypes = [vp] * 6 + [sz, *shape, i, vp]
        lib.na2d_block_workspace_bytes.argtypes = [*shape, i]
        lib.na2d_block_workspace_bytes.restype = sz
        lib.na2d_block_forward.argtypes = [vp] * 8 + [sz, *shape, i, vp]
        lib.na_forward_nd.argtypes = [vp] * 5 + [i] * 12 + [i, vp]
        lib.na2d_device_status.argtypes = [vp]
        lib.na2d_debug_timeout_probe.argtypes = [ctypes.c_uint, vp]
        lib.na_status_str.argtypes = [i]
        lib.na_status_str.restype = ctypes.c_char_p
        for name in ("na2d_qk_rpb", "na2d_softmax", "na2d_av", "na2d_forward",
                     "na2d_forward_host", "na2d_forward_host_noalloc", "na2d_forward_kernel", "na2d_device_status",
                     "na2d_debug_timeout_probe", "na2d_backward", "na2d_sasa_forward", "na2d_block_forward",
                     "na_forward_nd"):
            getattr(lib, name).restype = i
        _lib = lib
        return lib


def status_str(status: int) -> str:
    return load_library().na_status_str(status).decode()


def _check(status: int, what: str):
    if status != NA_OK:
        raise NA2DError(status, what)


def _stream(t: torch.Tensor | None = None):
    dev = t.device if t is not None else torch.device("cuda")
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _dims(q: torch.Tensor):
    if q.dim() != 5:
        raise ValueError("q/k/v must be [B, heads, H, W, d]")
    return tuple(int(x) for x in q.shape)


def forward(q, k, v, rpb, ksize: int, out=None):
    """Fused NA forward (na2d_forward): returns out [B, heads, H, W, d]."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    if rpb is not None:
        _need(rpb, "rpb", q.dtype)
    B, heads, H, W, d = _dims(q)
    out = torch.empty_like(q) if out is None else out
    _need(out, "out", q.dtype)
    _check(load_library().na2d_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(rpb), _ptr(out),
                                       B, heads, H, W, d, ksize, _DT[q.dtype], _stream(q)),
           "na2d_forward")
    return out


def qk_rpb(q, k, rpb, ksize: int, attn=None):
    """Unscaled Eq. (2) logits (na2d_qk_rpb): float32 [B, heads, H, W, ksize^2]."""
    _need(q, "q")
    _need(k, "k", q.dtype)
    if rpb is not None:
        _need(rpb, "rpb", q.dtype)
    B, heads, H, W, d = _dims(q)
    if attn is None:
        attn = torch.empty((B, heads, H, W, ksize * ksize), device=q.device, dtype=torch.float32)
    _need(attn, "attn", torch.float32)
    _check(load_library().na2d_qk_rpb(_ptr(q), _ptr(k), _ptr(rpb), _ptr(attn), B, heads, H, W, d,
                                      ksize, _DT[q.dtype], _stream(q)), "na2d_qk_rpb")
    return attn


def softmax_(attn, ksize: int, scale: float):
    """In-place softmax(scale * attn) over the last axis (na2d_softmax)."""
    _need(attn, "attn", torch.float32)
    B, heads, H, W, kk = (int(x) for x in attn.shape)
    if kk != ksize * ksize:
        raise ValueError("attn last axis must be ksize^2")
    _check(load_library().na2d_softmax(_ptr(attn), B, heads, H, W, ksize, float(scale),
                                       _stream(attn)), "na2d_softmax")
    return attn


def av(attn, v, ksize: int, out=None):
    """Eqs. (3)-(4) with given weights (na2d_av): out [B, heads, H, W, d]."""
    _need(attn, "attn", torch.float32)
    _need(v, "v")
    B, heads, H, W, d = _dims(v)
    out = torch.empty_like(v) if out is None else out
    _need(out, "out", v.dtype)
    _check(load_library().na2d_av(_ptr(attn), _ptr(v), _ptr(out), B, heads, H, W, d, ksize,
                                  _DT[v.dtype], _stream(v)), "na2d_av")
    return out


def backward(q, k, v, rpb, dout, ksize: int, with_rpb_grad: bool = True, workspace=None):
    """Gradients of a scalar loss through the NA forward (na2d_backward):
    returns (dq, dk, dv, drpb), drpb float32 [heads, 2k-1, 2k-1] or None."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (dout, "dout")):
        _need(t, n, q.dtype)
    if rpb is not None:
        _need(rpb, "rpb", q.dtype)
    B, heads, H, W, d = _dims(q)
    lib = load_library()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    drpb = (torch.empty((heads, 2 * ksize - 1, 2 * ksize - 1), device=q.device, dtype=torch.float32)
            if with_rpb_grad else None)
    need = int(lib.na2d_backward_workspace_bytes(B, heads, H, W, d, ksize, _DT[q.dtype]))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace")
    _check(lib.na2d_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(rpb), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                             _ptr(drpb), _ptr(workspace), workspace.numel() * workspace.element_size(),
                             B, heads, H, W, d, ksize, _DT[q.dtype], _stream(q)), "na2d_backward")
    return dq, dk, dv, drpb


def sasa_forward(q, k, v, rpb, ksize: int, out=None, workspace=None):
    """SASA, the centred window over a zero-padded map (na2d_sasa_forward):
    returns out [B, heads, H, W, d]."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    if rpb is not None:
        _need(rpb, "rpb", q.dtype)
    B, heads, H, W, d = _dims(q)
    out = torch.empty_like(q) if out is None else out
    _need(out, "out", q.dtype)
    lib = load_library()
    need = int(lib.na2d_sasa_workspace_bytes(B, heads, H, W, d, ksize, _DT[q.dtype]))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace")
    _check(lib.na2d_sasa_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(rpb), _ptr(out), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), B, heads, H, W, d, ksize,
                                 _DT[q.dtype], _stream(q)), "na2d_sasa_forward")
    return out


def block_forward(x, wqkv, bqkv, wo, bo, rpb, heads: int, ksize: int, y=None, workspace=None):
    """An NA block (na2d_block_forward): y = NA(x Wqkv + bqkv) Wo + bo, x and y
    [B, H, W, heads * dh]."""
    for t, n in ((x, "x"), (wqkv, "wqkv"), (wo, "wo")):
        _need(t, n, x.dtype)
    for t, n in ((bqkv, "bqkv"), (bo, "bo"), (rpb, "rpb")):
        if t is not None:
            _need(t, n, x.dtype)
    if x.dim() != 4:
        raise ValueError("x must be [B, H, W, C]")
    B, H, W, C = (int(s) for s in x.shape)
    if C % heads:
        raise ValueError("C must be a multiple of heads")
    dh = C // heads
    y = torch.empty_like(x) if y is None else y
    _need(y, "y", x.dtype)
    lib = load_library()
    need = int(lib.na2d_block_workspace_bytes(B, H, W, heads, dh, ksize, _DT[x.dtype]))
    if need == 0:
        raise NA2DError(NA_ERR_INVALID_ARG, "na2d_block_forward")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    _need(workspace, "workspace")
    _check(lib.na2d_block_forward(_ptr(x), _ptr(wqkv), _ptr(bqkv), _ptr(wo), _ptr(bo), _ptr(rpb), _ptr(y),
                                  _ptr(workspace), workspace.numel() * workspace.element_size(), B, H, W, heads, dh,
                                  ksize, _DT[x.dtype], _stream(x)), "na2d_block_forward")
    return y


def forward_nd(q, k, v, rpb, ks, dilation=None, out=None):
    """NA over the 1-3 spatial axes of q [B, heads, *spatial, d] with per-axis
    kernel sizes ks and dilations (na_forward_nd)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    if rpb is not None:
        _need(rpb, "rpb", q.dtype)
    nsp = q.dim() - 3
    if nsp not in (1, 2, 3):
        raise ValueError("q must be [B, heads, *spatial, d] with 1-3 spatial axes")
    ks = tuple(ks) if hasattr(ks, "__len__") else (ks,) * nsp
    dilation = tuple(dilation) if dilation is not None else (1,) * nsp
    B, heads, d = int(q.shape[0]), int(q.shape[1]), int(q.shape[-1])
    L = (1,) * (3 - nsp) + tuple(int(x) for x in q.shape[2:-1])
    kk = (1,) * (3 - nsp) + ks
    dl = (1,) * (3 - nsp) + dilation
    out = torch.empty_like(q) if out is None else out
    _need(out, "out", q.dtype)
    _check(load_library().na_forward_nd(_ptr(q), _ptr(k), _ptr(v), _ptr(rpb), _ptr(out), B, heads, *L, d, *kk, *dl,
                                        _DT[q.dtype], _stream(q)), "na_forward_nd")
    return out


def host_workspace_bytes(B, heads, H, W, d, ksize, dtype) -> int:
    return int(load_library().na2d_forward_host_workspace_bytes(B, heads, H, W, d, ksize, _DT[dtype]))


def forward_host(q_host, k_host, v_host, rpb_host, out_host, ksize: int, workspace, stream=None):
    """na2d_forward_host: host tensors in and out, a caller-owned device workspace."""
    B, heads, H, W, d = _dims(q_host)
    for t in (q_host, k_host, v_host, out_host) + ((rpb_host,) if rpb_host is not None else ()):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("host buffers must be contiguous CPU tensors")
    _need(workspace, "workspace")
    st = ctypes.c_void_p(stream.cuda_stream) if stream is not None else _stream(workspace)
    _check(load_library().na2d_forward_host(
        _ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(rpb_host), _ptr(out_host), _ptr(workspace),
        workspace.numel() * workspace.element_size(), B, heads, H, W, d, ksize, _DT[q_host.dtype], st),
        "na2d_forward_host")
    return out_host


def forward_host_noalloc(q_host, k_host, v_host, rpb_host, out_host, ksize: int, stream=None):
    """na2d_forward_host_noalloc: host tensors in and out, staged in the
    library's own fixed device array, for callers that cannot allocate device
    memory; shapes needing more than NOALLOC_SCRATCH_BYTES are rejected."""
    B, heads, H, W, d = _dims(q_host)
    for t in (q_host, k_host, v_host, out_host) + ((rpb_host,) if rpb_host is not None else ()):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("host buffers must be contiguous CPU tensors")
    st = ctypes.c_void_p(stream.cuda_stream) if stream is not None else _stream()
    _check(load_library().na2d_forward_host_noalloc(
        _ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(rpb_host), _ptr(out_host), B, heads, H, W, d, ksize,
        _DT[q_host.dtype], st), "na2d_forward_host_noalloc")
    return out_host


NOALLOC_SCRATCH_BYTES = 64 << 20  # NA2D_NOALLOC_SCRATCH_BYTES of include/na2d.h


def forward_kernel(B, heads, H, W, d, ksize, dtype) -> int:
    """1 if na2d_forward runs the tensor-core kernel for these arguments, 0 for SIMT."""
    return int(load_library().na2d_forward_kernel(B, heads, H, W, d, ksize, _DT[dtype]))


def device_status(stream=None) -> int:
    st = ctypes.c_void_p(stream.cuda_stream) if stream is not None else _stream()
    return int(load_library().na2d_device_status(st))


def debug_timeout_probe(timeout_us: int, stream=None) -> int:
    st = ctypes.c_void_p(stream.cuda_stream) if stream is not None else _stream()
    return int(load_library().na2d_debug_timeout_probe(int(timeout_us), st))
