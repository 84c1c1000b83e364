"""Parity of the Spatial SwiGLU stencil (gtr_sswiglu_dwconv) with the fp64 oracle:
SiLU(xg) * DWConv3x3(xv), zero padding, every dtype, ragged grids (tiles that cross the
grid edge), with and without bias.  Bound: max |z - z_ref| <= tol * rms(z_ref), tol =
1e-2 for 16-bit data (the output's own rounding is 2^-9 relative for bf16) and 1e-5 for
fp32."""
import numpy as np
import pytest
import torch

import gated_token_recurrence_b200 as gtr
import oracle
from gtr_inputs import STENCILS, StencilWorkload, make_stencil_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 1e-2, "bf16": 1e-2}


def check(s: StencilWorkload, seed: int):
    dev = torch.device("cuda:0")
    xg, xv, w, b = make_stencil_inputs(s, seed)
    ref = oracle.sswiglu_dwconv(xg, xv, w, b, s.H, s.W)
    out = gtr.sswiglu_dwconv(xg.to(dev), xv.to(dev), w.to(dev), None if b is None else b.to(dev), grid=(s.H, s.W))
    torch.cuda.synchronize()
    o = out.to("cpu", torch.float64).numpy()
    assert np.isfinite(o).all()
    err = float(np.abs(o - ref).max() / np.sqrt(np.mean(ref ** 2)))
    assert err <= TOL[s.dtype], f"{s.name}: max err / rms = {err:.3e}"


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
