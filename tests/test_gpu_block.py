"""Parity of the GTR block call (gtr_gla_block_fwd) with the fp64 oracle: the low-rank
gate producer (log gamma = logsigmoid(z W2 + b) / tau, fused into the loads), the
RMSNorm + SiLU output-gate epilogue, and both together, in every plan of the fused
kernel and on the split path, all four directions.

Criterion without the output gate: max |y - y_ref| <= tol * rms(y_ref), tol = 1e-2 for
fp16/bf16 inputs and 1e-5 for fp32 inputs (the bound of the plain operation).

With the output gate the bound is carried through the epilogue.  RMSNorm divides each
token-head row by its own rms, so the normalised output has unit rms per row and the GLA
output's bound becomes tol in those units; the gate then multiplies each element by
w_j * SiLU(gate_ij), and its error with it.  So the check is
    max_ij |y - y_ref|_ij / max(|w_j SiLU(gate_ij)|, 1) <= tol.
(Against rms(y_ref) instead, the heavy tail of the product -- |SiLU(g)| up to ~4 where
rms(SiLU(g)) ~ 0.6 -- would tighten the plain bound several times over.)
"""
import numpy as np
import pytest
import torch

import gated_token_recurrence_b200 as gtr
import oracle
from gtr_inputs import (WORKLOADS, Workload, make_gate_epilogue_inputs, make_inputs,
                        make_lowrank_gate_inputs)

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 1e-2, "bf16": 1e-2}
PATHS = ["auto", "split", "fused", "fused_sequential"]
# one cluster per sequence; segments exchanging summaries; one CTA per sequence
SHAPES = {"cluster": (1, 6, 40, 40), "segmented": (1, 2, 128, 112), "stream": (13, 6, 8, 16)}


def rel_err(out: torch.Tensor, ref: np.ndarray) -> float:
    o = out.detach().to("cpu", torch.float64).numpy()
    assert np.isfinite(o).all(), "non-finite output"
    return float(np.abs(o - ref).max() / np.sqrt(np.mean(ref ** 2)))


def run_block(w, d, seed, path, lowrank=True, gated=True, rank=16, offset=None, out_dtype=None):
    dev = torch.device("cuda:0")
    q, k, v, lg = make_inputs(w, seed)
    kw = {}
    if lowrank:
        z, w2, b = make_lowrank_gate_inputs(w, seed, rank=rank, offset=offset)
        kw.update(gate_z=z.to(dev), gate_w2=w2.to(dev), gate_b=b.to(dev), gate_tau=16.0)
    else:
        kw.update(log_gamma=lg.to(dev))
    if gated:
        og, nw, eps = make_gate_epilogue_inputs(w, seed)
        kw.update(out_gate=og.to(dev), norm_w=nw.to(dev), norm_eps=eps)
    out = None
    if out_dtype is not None:
        out = torch.empty((w.B, w.L, w.heads, w.d_v), dtype=out_dtype, device=dev)
    y = gtr.gla_block_fwd(q.to(dev), k.to(dev), v.to(dev), grid=(w.H, w.W), direction=d, out=out, path=path, **kw)
    torch.cuda.synchronize()
    # the oracle, on the same bytes
    if lowrank:
        ref = oracle.gla_fwd_lowrank(q, k, v, z, w2, b, 16.0, w.H, w.W, d)
    else:
        ref = oracle.gla_fwd(q, k, v, lg, w.H, w.W, d)
    gate_factor = None
    if gated:
        ref = oracle.rmsnorm_silu_gate(ref, og, nw, eps)
        g = og.double().numpy()
        gate_factor = np.abs(nw.double().numpy() * g / (1.0 + np.exp(-g)))
    return y, ref, gate_factor


def gated_err(out: torch.Tensor, ref: np.ndarray, gate_factor: np.ndarray) -> float:
    """max |y - y_ref| in units of the normalised output, per element divided by the gate
    factor |w_j SiLU(gate_ij)| where that exceeds 1 (see the module docstring)."""
    o = out.detach().to("cpu", torch.float64).numpy()
    assert np.isfinite(o).all(), "non-finite output"
    return float((np.abs(o - ref) / np.maximum(gate_factor, 1.0)).max())


def check_block(w, d, seed, path, **kw):
    y, ref, gf = run_block(w, d, seed, path, **kw)
    err = rel_err(y, ref) if gf is None else gated_err(y, ref, gf)
    assert err <= TOL[w.dtype], f"{w.name} dir={d} path={path} {kw}: max err = {err:.3e}"


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("plan", list(SHAPES))
@pytest.mark.parametrize("pieces", ["lowrank", "gated", "both"])
def test_block_pieces_in_every_plan(pieces, plan, path):
    B, heads, H, W = SHAPES[plan]
    w = Workload("blk", B=B, heads=heads, H=H, W=W, dtype="f16", scale=0.5, index=9)
    for d in range(4):
        check_block(w, d, 8100 + d, path, lowrank=pieces != "gated", gated=pieces != "lowrank")


@pytest.mark.parametrize("name", ["640", "1024", "2048"])
def test_block_on_the_workloads(name):
    """The full block (low-rank gates with the workload's gate offset, output gate) on the
    workload grids; 2048^2 keeps its strongly retentive gates (bias +4)."""
    w = WORKLOADS[name]
    for d in w.directions:
        check_block(w, d, w.seed(d) + 64, "auto")


@pytest.mark.parametrize("rank", [8, 16])
def test_block_gate_ranks(rank):
    w = Workload("rk", B=2, heads=3, H=24, W=40, dtype="bf16", index=9)
    for d in range(4):
        check_block(w, d, 8200 + rank + d, "auto", rank=rank, gated=False)


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
def test_block_key_width_32_and_dtypes(dtype):
    for dk in (32, 64):
        w = Workload("dt", B=1, heads=4, H=32, W=48, d_k=dk, dtype=dtype, index=9)
        for d in range(4):
            check_block(w, d, 8300 + dk + d, "auto")


@pytest.mark.parametrize("shape", [(1, 1, 1, 1), (1, 3, 7, 9), (2, 2, 5, 13), (1, 2, 33, 31), (2, 3, 65, 1)])
def test_block_ragged_shapes(shape):
    B, heads, H, W = shape
    w = Workload("oddb", B=B, heads=heads, H=H, W=W, dtype="bf16", index=9)
    for d in range(4):
        for path in ("auto", "fused"):
            check_block(w, d, 8400 + H + W + d, path)


def test_block_with_caller_workspace_in_a_graph():
    """The block call with a caller workspace, captured in a CUDA graph and replayed."""
    w = WORKLOADS["640"].with_(heads=2)
    dev = torch.device("cuda:0")
    q, k, v, _ = make_inputs(w, 8500)
    z, w2, b = make_lowrank_gate_inputs(w, 8500)
    og, nw, eps = make_gate_epilogue_inputs(w, 8500)
    ref = oracle.rmsnorm_silu_gate(oracle.gla_fwd_lowrank(q, k, v, z, w2, b, 16.0, w.H, w.W, 2), og, nw, eps)
    g = og.double().numpy()
    gf = np.abs(nw.double().numpy() * g / (1.0 + np.exp(-g)))
    t = dict(gate_z=z.to(dev), gate_w2=w2.to(dev), gate_b=b.to(dev), out_gate=og.to(dev), norm_w=nw.to(dev),
             norm_eps=eps)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    ws = gtr.new_workspace(w.B, w.heads, w.H, w.W, in_dtype=gtr.F16, device=dev)
    out = torch.empty((w.B, w.L, w.heads, w.d_v), dtype=torch.float16, device=dev)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        gtr.gla_block_fwd(qd, kd, vd, grid=(w.H, w.W), direction=2, out=out, workspace=ws, stream=s, **t)
    torch.cuda.synchronize()
    out.fill_(float("nan"))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        gtr.gla_block_fwd(qd, kd, vd, grid=(w.H, w.W), direction=2, out=out, workspace=ws, stream=s, **t)
    with torch.cuda.stream(s):
        graph.replay()
    torch.cuda.synchronize()
    assert gated_err(out, ref, gf) <= 1e-2
    assert gtr.read_error(ws) == 0
    del graph
