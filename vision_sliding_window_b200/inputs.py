"""Seeded synthetic inputs for 2D neighborhood attention.

This module holds only data generation: shapes, seeds and value
distributions.  It contains none of the operator's arithmetic, so both the
CUDA path's tests and the fp64 oracle can take their inputs from it.

Each workload stands in for a NAT feature map (Neighborhood Attention
Transformer, Sec. 3.3 / Sec. 4: a 224x224 image gives 56/28/14/7 maps;
detection and segmentation inputs give maps of a few hundred pixels).
q, k, v are drawn from N(0, 1) in fp32 (scaled by 1/sqrt(d) where the
workload says so) and the relative-position table from N(0, 0.02^2), from
one CPU generator seeded per workload, in the order q, k, v, rpb; then each
tensor is rounded to the workload's dtype.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    heads: int
    H: int
    W: int
    d: int
    ks: int
    dtype: str  # "f32" | "f16" | "bf16"
    qkv_scale: float = 1.0
    rpb_std: float = 0.02
    seed: int = 0
    note: str = field(default="", compare=False)

    @property
    def queries(self) -> int:
        return self.B * self.heads * self.H * self.W

    @property
    def query_neighbours(self) -> int:
        return self.queries * self.ks * self.ks

    @property
    def elem_bytes(self) -> int:
        return torch.tensor([], dtype=DTYPES[self.dtype]).element_size()

    @property
    def io_bytes(self) -> int:
        """Algorithmic HBM bytes of one forward: read q, k, v and the table once,
        write out once."""
        tensor = self.queries * self.d * self.elem_bytes
        rpb = self.heads * (2 * self.ks - 1) ** 2 * self.elem_bytes
        return 4 * tensor + rpb

    @property
    def flops(self) -> int:
        """Algorithmic FLOPs: the NA part of the complexity model, 2*h*w*d*k^2
        multiply-adds per head (logits and weighted sum), counted as 2 FLOPs each."""
        return 4 * self.queries * self.ks * self.ks * self.d

    def shape(self):
        return (self.B, self.heads, self.H, self.W, self.d)


def _sweep(ks: int) -> Workload:
    return Workload(f"sweep_k{ks}", 8, 4, 128, 128, 64, ks, "f16", qkv_scale=64 ** -0.5,
                    note="kernel-size sweep, q/k/v scaled by 1/sqrt(d)")


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", 1, 1, 14, 14, 32, 7, "f32", note="oracle check"),
        Workload("tiny_sa", 1, 1, 7, 7, 32, 7, "f32", note="k = H = W: equals full self-attention"),
        Workload("stage1", 32, 2, 56, 56, 32, 7, "bf16", note="NAT-Tiny level-1 map"),
        Workload("stage3", 128, 8, 14, 14, 32, 7, "f16", note="NAT-Tiny level-3 map"),
        Workload("stage4", 128, 16, 7, 7, 32, 7, "f16", note="NAT-Tiny level-4 map, window = whole map"),
        Workload("hires_k7", 2, 4, 256, 256, 32, 7, "bf16", note="dense-prediction map"),
        Workload("hires_k13", 2, 4, 256, 256, 32, 13, "bf16", note="dense-prediction map"),
    ]
    + [_sweep(k) for k in (3, 5, 7, 9, 11, 13)]
}


def make_inputs(B: int, heads: int, H: int, W: int, d: int, ks: int, dtype="bf16", *,
                seed: int = 0, qkv_scale: float = 1.0, rpb_std: float = 0.02,
                with_rpb: bool = True):
    """Returns CPU tensors (q, k, v, rpb) in `dtype`; rpb is None when with_rpb is False."""
    tdt = DTYPES[dtype] if isinstance(dtype, str) else dtype
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    shp = (B, heads, H, W, d)
    q = torch.randn(shp, generator=g, dtype=torch.float32)
    k = torch.randn(shp, generator=g, dtype=torch.float32)
    v = torch.randn(shp, generator=g, dtype=torch.float32)
    rpb = torch.randn((heads, 2 * ks - 1, 2 * ks - 1), generator=g, dtype=torch.float32) * rpb_std
    if qkv_scale != 1.0:
        q, k, v = q * qkv_scale, k * qkv_scale, v * qkv_scale
    return (q.to(tdt), k.to(tdt), v.to(tdt), rpb.to(tdt) if with_rpb else None)


def workload_inputs(w: Workload, with_rpb: bool = True):
    return make_inputs(w.B, w.heads, w.H, w.W, w.d, w.ks, w.dtype, seed=w.seed,
                       qkv_scale=w.qkv_scale, rpb_std=w.rpb_std, with_rpb=with_rpb)


def sample_points(w: Workload, n: int, seed: int = 1):
    """n query points (b, h, i, j): all four corners and edge midpoints of the
    first and last (b, h), plus uniformly drawn points, as an int64 [n, 4] tensor."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    fixed = []
    for b, h in ((0, 0), (w.B - 1, w.heads - 1)):
        for i in (0, w.H // 2, w.H - 1):
            for j in (0, w.W // 2, w.W - 1):
                fixed.append((b, h, i, j))
    pts = torch.tensor(fixed, dtype=torch.int64)
    extra = max(0, n - len(fixed))
    if extra:
        rnd = torch.stack([
            torch.randint(0, w.B, (extra,), generator=g),
            torch.randint(0, w.heads, (extra,), generator=g),
            torch.randint(0, w.H, (extra,), generator=g),
            torch.randint(0, w.W, (extra,), generator=g),
        ], dim=1)
        pts = torch.cat([pts, rnd])
    return pts[:max(n, len(fixed))]


def make_block_inputs(B: int, H: int, W: int, heads: int, dh: int, ks: int, dtype="bf16", *, seed: int = 0):
    """Synthetic weights and input of an NA block (x [B, H, W, C], Wqkv [C, 3C],
    bqkv [3C], Wo [C, C], bo [C], rpb [heads, 2ks-1, 2ks-1], C = heads * dh):
    x ~ N(0, 1), weights ~ N(0, 1/C), biases ~ N(0, 0.1^2), rpb ~ N(0, 0.02^2),
    from one CPU generator in that order, then rounded to `dtype`."""
    tdt = DTYPES[dtype] if isinstance(dtype, str) else dtype
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    C = heads * dh
    x = torch.randn((B, H, W, C), generator=g)
    wqkv = torch.randn((C, 3 * C), generator=g) / C ** 0.5
    bqkv = torch.randn(3 * C, generator=g) * 0.1
    wo = torch.randn((C, C), generator=g) / C ** 0.5
    bo = torch.randn(C, generator=g) * 0.1
    rpb = torch.randn((heads, 2 * ks - 1, 2 * ks - 1), generator=g) * 0.02
    return tuple(t.to(tdt) for t in (x, wqkv, bqkv, wo, bo, rpb))
