"""Parity of the Spatial SwiGLU stencil (gtr_sswiglu_dwconv) with the fp64 oracle:
SiLU(xg) * DWConv3x3(xv), zero padding, every dtype, ragged grids (tiles that cross the
grid edge), with and without bias.

Bound, derived from the arithmetic: the kernel reads the inputs exactly, computes the
nine taps, the bias and SiLU in fp32 and rounds once to the output dtype, so per element
    |z - z_ref| <= u_out * |z_ref| + 1e-5 * rms(z_ref)
with u_out the output dtype's unit roundoff (2^-8 bf16, 2^-11 fp16, 2^-24 fp32) and the
second term the fp32 arithmetic.  (Measured against rms(z_ref) alone, the bf16 rounding
of the heavy-tailed product would exceed 1e-2 by itself: max |z| is 10-20 rms.)"""
import numpy as np
import pytest
import torch

import gated_token_recurrence_b200 as gtr
import oracle
from gtr_inputs import STENCILS, StencilWorkload, make_stencil_inputs

pytestmark = pytest.mark.gpu

UNIT_ROUNDOFF = {"f32": 2.0 ** -24, "f16": 2.0 ** -11, "bf16": 2.0 ** -8}


def check(s: StencilWorkload, seed: int):
    dev = torch.device("cuda:0")
    xg, xv, w, b = make_stencil_inputs(s, seed)
    ref = oracle.sswiglu_dwconv(xg, xv, w, b, s.H, s.W)
    out = gtr.sswiglu_dwconv(xg.to(dev), xv.to(dev), w.to(dev), None if b is None else b.to(dev), grid=(s.H, s.W))
    torch.cuda.synchronize()
    o = out.to("cpu", torch.float64).numpy()
    assert np.isfinite(o).all()
    bound = UNIT_ROUNDOFF[s.dtype] * np.abs(ref) + 1e-5 * np.sqrt(np.mean(ref ** 2))
    worst = float((np.abs(o - ref) / bound).max())
    assert worst <= 1.0, f"{s.name}: max |z - z_ref| / bound = {worst:.3f}"


@pytest.mark.parametrize("name", list(STENCILS))
def test_stencil_workloads(name):
    check(STENCILS[name], 9100)


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("shape", [(1, 1, 1), (2, 3, 5), (1, 9, 17), (1, 40, 40), (3, 13, 31), (1, 1, 70)])
@pytest.mark.parametrize("bias", [True, False])
def test_stencil_ragged_grids(shape, dtype, bias):
    B, H, W = shape
    s = StencilWorkload("odd", B=B, H=H, W=W, C=128, dtype=dtype, bias=bias)
    check(s, 9200 + H * 100 + W)
