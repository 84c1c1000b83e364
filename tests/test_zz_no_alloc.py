"""gtr_gla_fwd_noalloc: the allocation-free entry point, through the C ABI.

It exists for callers that may not call cudaMalloc (an inference-engine
plugin limited to memory handed out at build time, a real-time loop that
cannot afford cudaMalloc's implicit device synchronisation).  Its scratch is a
fixed array inside the library.  These checks run it twice in a row (the
second call finds the first call's leftovers in the shared array) and compare
each output with the existing entry point on the same path (gtr_gla_fwd_ex
with a workspace the test allocates) and with the fp64 oracle; they check that
a call allocates no device memory, and that a problem too big for the array is
refused.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import gated_token_recurrence_b200 as gtr
import oracle
from gtr_inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 1e-2, "bf16": 1e-2}
CODE = {"f32": gtr.F32, "f16": gtr.F16, "bf16": gtr.BF16}


def call_noalloc(w, tensors, out, direction):
    q, k, v, lg = tensors
    return gtr.lib.gtr_gla_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), lg.data_ptr(),
                                       out.data_ptr(), w.B, w.heads, w.H, w.W, w.d_k, w.d_v,
                                       direction, CODE[w.dtype], CODE[w.out_dtype],
                                       torch.cuda.current_stream().cuda_stream)


def err_over_rms(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.abs(a - b).max() / np.sqrt(np.mean(b ** 2)))


def test_noalloc_matches_the_split_entry_and_the_oracle_on_two_calls_in_a_row():
    dev = torch.device("cuda:0")
    cases = [(WORKLOADS["640"], 1, 811), (WORKLOADS["1024"].with_(heads=4), 3, 812)]
    prepared = []
    for w, d, seed in cases:
        host = make_inputs(w, seed)
        t = tuple(x.to(dev) for x in host)
        out = torch.full((w.B, w.L, w.heads, w.d_v), float("nan"),
                         dtype=gtr.default_out_dtype(t[0].dtype), device=dev)
        prepared.append((w, d, host, t, out))
    # two calls back to back, no synchronisation between them
    for w, d, _, t, out in prepared:
        assert call_noalloc(w, t, out, d) == 0
    torch.cuda.synchronize()
    for w, d, host, t, out in prepared:
        ws = gtr.new_workspace(w.B, w.heads, w.H, w.W, in_dtype=CODE[w.dtype], path="split", device=dev)
        ref_gpu = gtr.gla_fwd(*t, grid=(w.H, w.W), direction=d, path="split", workspace=ws)
        torch.cuda.synchronize()
        a = out.double().cpu().numpy()
        b = ref_gpu.double().cpu().numpy()
        assert np.isfinite(a).all()
        # the same kernels on the same inputs: within the tolerance, and in fact identical
        assert err_over_rms(a, b) <= TOL[w.dtype], w.name
        assert torch.equal(out, ref_gpu), f"{w.name}: noalloc and gtr_gla_fwd_ex(split) differ"
        ref = oracle.gla_fwd(*host, w.H, w.W, d)
        err = err_over_rms(a, ref)
        assert err <= TOL[w.dtype], f"{w.name}: max err / rms against the oracle {err:.3e}"
    assert gtr.read_error() == 0


def test_noalloc_allocates_no_device_memory():
    """Free device memory is unchanged across calls on ever larger problems, up to the
    array's limit of 634 chunk units (a growing workspace would take 2 MiB or more)."""
    dev = torch.device("cuda:0")
    shapes = [(1, 1, 8, 64), (1, 2, 32, 64), (1, 3, 64, 100), (1, 2, 64, 317)]  # ... 634 units
    runs = []
    for B, heads, H, W in shapes:
        w = WORKLOADS["640"].with_(B=B, heads=heads, H=H, W=W)
        t = tuple(x.to(dev) for x in make_inputs(w, 900 + W))
        runs.append((w, t, torch.empty((B, H * W, heads, 64), dtype=torch.float16, device=dev)))
    assert call_noalloc(runs[0][0], runs[0][1], runs[0][2], 0) == 0  # the kernels are loaded
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info(dev)[0]
    for w, t, out in runs:
        assert call_noalloc(w, t, out, 2) == 0
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info(dev)[0]
    assert abs(free0 - free1) < (2 << 20), f"device memory changed by {free0 - free1} bytes"


def test_noalloc_refuses_problems_beyond_its_scratch():
    w = WORKLOADS["2048"]  # 6 heads x 256 chunks = 1536 units > 634
    dev = torch.device("cuda:0")
    t = tuple(torch.empty(16, dtype=torch.float16 if i < 3 else torch.float32, device=dev)
              for i in range(4))
    out = torch.empty(16, dtype=torch.float16, device=dev)
    assert call_noalloc(w, t, out, 0) == 5  # GTR_ERR_WORKSPACE, nothing enqueued
