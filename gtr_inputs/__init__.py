"""Seeded synthetic inputs and the named workloads.

This module holds no arithmetic of the operation itself; it only draws the
inputs (and the gate distribution, which in GTR comes from an upstream
low-rank projection, ``gamma = sigmoid(.)^(1/tau)`` with tau = 16 - digest
page paper.rainbus.top, section "Core method").  Both the CUDA path's tests
and the oracle's tests draw from here, so the two sides see identical bytes.

Recipe (the same for every workload): a CPU ``torch.Generator`` seeded with
``seed`` draws q, k, v, g in that order, each fp32 N(0, 1) of shape
[B, L, heads, d]; q, k, v are multiplied by ``scale`` and rounded to the
storage dtype (round-to-nearest-even); ``log_gamma = logsigmoid(g + offset) / tau`` (tau = 16 unless a test asks for
stronger gates)
stays fp32.  The grids are the stride-16 patch grids of the images the GTR
pages evaluate (640^2 -> 40x40, 1024^2 -> 64x64, 2048^2 -> 128x128,
1280x768 -> 80 wide by 48 high).  No public dataset is involved.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import List, Optional

import torch
import torch.nn.functional as F

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
# output dtype that goes with each input dtype (bf16 output would lose the
# 1e-2 * rms accuracy budget on its own, so bf16 inputs produce fp32 output)
OUT_DTYPE = {"f32": "f32", "f16": "f16", "bf16": "f32"}
DIRECTION_NAMES = ("l2r", "r2l", "t2b", "b2t")


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    heads: int
    H: int
    W: int
    d_k: int = 64
    d_v: int = 64
    dtype: str = "f16"
    scale: float = 1.0
    gate_offset: float = 0.0
    gate_tau: float = 16.0
    directions: tuple = (0,)
    calls: int = 1
    index: int = 0
    note: str = ""

    @property
    def L(self) -> int:
        return self.H * self.W

    @property
    def out_dtype(self) -> str:
        return OUT_DTYPE[self.dtype]

    @property
    def token_heads(self) -> int:
        return self.B * self.L * self.heads

    def direction_of_call(self, call: int) -> int:
        return self.directions[call % len(self.directions)]

    def seed(self, direction: int, call: int = 0) -> int:
        return 1000 * self.index + 10 * direction + call

    def algorithmic_bytes(self) -> int:
        """HBM bytes one call must move: read q, k, v, log_gamma; write out."""
        es = torch.finfo(DTYPES[self.dtype]).bits // 8
        eo = torch.finfo(DTYPES[self.out_dtype]).bits // 8
        per = (2 * self.d_k + self.d_v) * es + self.d_k * 4 + self.d_v * eo
        return self.token_heads * per

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", B=1, heads=2, H=16, W=16, dtype="f32", scale=1.0,
                 directions=(0,), index=0,
                 note="tiny oracle check, fp32, 16x16 grid"),
        Workload("640", B=1, heads=6, H=40, W=40, dtype="f16", scale=0.5,
                 directions=(0, 1, 2, 3), index=1,
                 note="640^2 image at stride 16 (1.6K tokens), fp16"),
        Workload("1024", B=1, heads=8, H=64, W=64, dtype="bf16", scale=1.0,
                 directions=(0, 1, 2, 3), index=2,
                 note="1024^2 image (4.1K tokens), bf16"),
        Workload("2048", B=1, heads=6, H=128, W=128, dtype="f16", scale=0.5,
                 gate_offset=4.0, directions=(0, 3), index=3,
                 note="2048^2 image (16.4K tokens), fp16, strongly retentive gates"),
        Workload("stack", B=8, heads=6, H=48, W=80, dtype="bf16", scale=1.0,
                 directions=(0, 1, 2, 3), calls=12, index=4,
                 note="batched 1280x768 stack (grid 80 wide, 48 high), bf16, 12 calls"),
    ]
}


def make_inputs(w: Workload, seed: int, device: Optional[str] = None):
    """Draw (q, k, v, log_gamma) for workload ``w`` from a CPU generator seeded with ``seed``."""
    gen = torch.Generator(device="cpu").manual_seed(int(seed))
    shape_k = (w.B, w.L, w.heads, w.d_k)
    shape_v = (w.B, w.L, w.heads, w.d_v)
    q = torch.randn(shape_k, generator=gen, dtype=torch.float32)
    k = torch.randn(shape_k, generator=gen, dtype=torch.float32)
    v = torch.randn(shape_v, generator=gen, dtype=torch.float32)
    g = torch.randn(shape_k, generator=gen, dtype=torch.float32)
    dt = DTYPES[w.dtype]
    q = (q * w.scale).to(dt)
    k = (k * w.scale).to(dt)
    v = (v * w.scale).to(dt)
    log_gamma = F.logsigmoid(g + w.gate_offset) / w.gate_tau
    if device is not None:
        q, k, v, log_gamma = (t.to(device) for t in (q, k, v, log_gamma))
    return q, k, v, log_gamma


def empty_out(w: Workload, device=None) -> torch.Tensor:
    return torch.empty((w.B, w.L, w.heads, w.d_v), dtype=DTYPES[w.out_dtype], device=device)


# ----------------------------------------------------------------------------- GTR block pieces
# The recipes below draw the extra inputs of the block-level calls; like make_inputs they
# hold no arithmetic of the method.  GTR-L's widths (0539edu.com appendix D.1.1): model
# dimension 384 over 6 heads, S-SwiGLU expansion ratio 4 (hidden width 1536; GTR-X 6).
GATE_RANK = 16   # rank of the gate factorisation (GTR digest page, "Core method")
GATE_TAU = 16.0  # gamma = sigmoid(.)^(1/tau)


def make_lowrank_gate_inputs(w: Workload, seed: int, rank: int = GATE_RANK, offset: Optional[float] = None):
    """(z, w2, bias) for the low-rank gate producer, fp32: z = x W1 ~ N(0, 1) [B, L, rank];
    W2 ~ N(0, 1/rank) [rank, heads * d_k], so that z W2 ~ N(0, 1) per entry like the
    direct gate recipe; bias = the workload's gate offset (default) [heads * d_k]."""
    gen = torch.Generator(device="cpu").manual_seed(int(seed) + 555)
    z = torch.randn((w.B, w.L, rank), generator=gen, dtype=torch.float32)
    w2 = torch.randn((rank, w.heads * w.d_k), generator=gen, dtype=torch.float32) / rank ** 0.5
    off = w.gate_offset if offset is None else offset
    bias = torch.full((w.heads * w.d_k,), float(off), dtype=torch.float32)
    return z, w2, bias


def make_gate_epilogue_inputs(w: Workload, seed: int):
    """(gate, weight, eps) for the RMSNorm + SiLU output gate: gate ~ N(0, 1) in the input
    dtype [B, L, heads, d_v]; weight ~ 1 + 0.1 N(0, 1) fp32 [d_v]; eps = 1e-6."""
    gen = torch.Generator(device="cpu").manual_seed(int(seed) + 777)
    gate = torch.randn((w.B, w.L, w.heads, w.d_v), generator=gen, dtype=torch.float32).to(DTYPES[w.dtype])
    weight = 1.0 + 0.1 * torch.randn((w.d_v,), generator=gen, dtype=torch.float32)
    return gate, weight, 1e-6


@dataclass(frozen=True)
class StencilWorkload:
    """Spatial SwiGLU stencil: the two projections X W_g, X W_v of an H x W token grid."""
    name: str
    B: int
    H: int
    W: int
    C: int
    dtype: str = "f16"
    bias: bool = True
    index: int = 0

    @property
    def L(self) -> int:
        return self.H * self.W

    def algorithmic_bytes(self) -> int:
        """HBM bytes one call must move: read xg and xv, write z (all in dtype), plus the
        3x3 weights and bias (fp32)."""
        es = torch.finfo(DTYPES[self.dtype]).bits // 8
        return 3 * self.B * self.L * self.C * es + self.C * 10 * 4

    def with_(self, **kw) -> "StencilWorkload":
        return replace(self, **kw)


STENCILS = {
    s.name: s
    for s in [
        # GTR-L hidden width 1536 on the 640^2 / 1024^2 / 2048^2 grids
        StencilWorkload("sw640", B=1, H=40, W=40, C=1536, dtype="f16", index=11),
        StencilWorkload("sw1024", B=1, H=64, W=64, C=1536, dtype="bf16", index=12),
        StencilWorkload("sw2048", B=1, H=128, W=128, C=1536, dtype="f16", index=13),
    ]
}


def make_stencil_inputs(s: StencilWorkload, seed: int):
    """(xg, xv, conv_w, conv_b): xg, xv ~ N(0, 1) in the stencil's dtype [B, L, C];
    3x3 depthwise weights ~ N(0, 1/9) fp32 [C, 3, 3]; bias ~ 0.1 N(0, 1) fp32 [C] (or None)."""
    gen = torch.Generator(device="cpu").manual_seed(int(seed))
    dt = DTYPES[s.dtype]
    xg = torch.randn((s.B, s.L, s.C), generator=gen, dtype=torch.float32).to(dt)
    xv = torch.randn((s.B, s.L, s.C), generator=gen, dtype=torch.float32).to(dt)
    conv_w = torch.randn((s.C, 3, 3), generator=gen, dtype=torch.float32) / 3.0
    conv_b = 0.1 * torch.randn((s.C,), generator=gen, dtype=torch.float32) if s.bias else None
    return xg, xv, conv_w, conv_b
