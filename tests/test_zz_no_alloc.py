"""gtr_gla_fwd_noalloc: the allocation-free entry point, through the C ABI.

It exists for callers that may not call cudaMalloc (an inference-engine
plugin limited to memory handed out at build time, a real-time loop that
cannot afford cudaMalloc's implicit device synchronisation).  Its scratch is a
fixed array inside the library, so these checks compare it with the ordinary
entry point, gtr_gla_fwd, on two calls in a row (the second call finds the
first call's leftovers in the shared array), and check that a problem too big
for the array is refused.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import gated_token_recurrence_b200 as gtr
from gtr_inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 1e-2, "bf16": 1e-2}


def noalloc():
    f = gtr.lib.gtr_gla_fwd_noalloc
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 9 + [ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


def call_noalloc(w, tensors, out, direction):
    q, k, v, lg = tensors
    return noalloc()(q.data_ptr(), k.data_ptr(), v.data_ptr(), lg.data_ptr(), out.data_ptr(),
                     w.B, w.heads, w.H, w.W, w.d_k, w.d_v, direction,
                     {"f32": gtr.F32, "f16": gtr.F16, "bf16": gtr.BF16}[w.dtype],
                     {"f32": gtr.F32, "f16": gtr.F16, "bf16": gtr.BF16}[w.out_dtype],
                     torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_gtr_gla_fwd_on_two_calls_in_a_row():
    dev = torch.device("cuda:0")
    cases = [(WORKLOADS["640"], 1, 811), (WORKLOADS["1024"].with_(heads=4), 3, 812)]
    prepared = []
    for w, d, seed in cases:
        t = tuple(x.to(dev) for x in make_inputs(w, seed))
        out = torch.full((w.B, w.L, w.heads, w.d_v), float("nan"),
                         dtype=gtr.default_out_dtype(t[0].dtype), device=dev)
        prepared.append((w, d, t, out))
    # two calls back to back, no synchronisation between them
    for w, d, t, out in prepared:
        assert call_noalloc(w, t, out, d) == 0
    torch.cuda.synchronize()
    for w, d, t, out in prepared:
        ref = gtr.gla_fwd(*t, grid=(w.H, w.W), direction=d)
        torch.cuda.synchronize()
        a = out.double().cpu().numpy()
        b = ref.double().cpu().numpy()
        assert np.isfinite(a).all()
        err = np.abs(a - b).max() / np.sqrt(np.mean(b ** 2))
        assert err <= TOL[w.dtype], f"{w.name}: {err:.3e}"


def test_noalloc_refuses_problems_beyond_its_scratch():
    w = WORKLOADS["2048"]  # 6 heads x 256 chunks = 1536 units > 636
    dev = torch.device("cuda:0")
    t = tuple(torch.empty(1, dtype=torch.float16 if i < 3 else torch.float32, device=dev)
              for i in range(4))
    out = torch.empty(1, dtype=torch.float16, device=dev)
    assert call_noalloc(w, t, out, 0) == 5  # GTR_ERR_WORKSPACE, nothing enqueued
