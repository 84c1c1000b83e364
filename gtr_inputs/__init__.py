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
