"""Python binding of libgtr.so (key-only gated linear attention forward, sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libgtr.so``.  PyTorch supplies device memory and streams.  There
is no CPU fallback: importing this package fails if the library is missing.

    import gated_token_recurrence_b200 as gtr
    out = gtr.gla_fwd(q, k, v, log_gamma, grid=(H, W), direction=gtr.L2R)

Tensors are [B, L, heads, d] (log_gamma fp32 [B, L, heads, d_k]), contiguous,
on the current CUDA device.  See include/gtr.h for the full contract.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgtr.so")

L2R, R2L, T2B, B2T = 0, 1, 2, 3
F32, F16, BF16 = 0, 1, 2
PATH_AUTO, PATH_SPLIT, PATH_FUSED, PATH_FUSED_SEQUENTIAL = 0, 1, 2, 3
PATHS = {"auto": PATH_AUTO, "split": PATH_SPLIT, "fused": PATH_FUSED,
         "fused_sequential": PATH_FUSED_SEQUENTIAL}
STATUS = {0: "GTR_OK", 1: "GTR_ERR_INVALID_ARG", 2: "GTR_ERR_UNSUPPORTED", 3: "GTR_ERR_CUDA",
          4: "GTR_ERR_TIMEOUT", 5: "GTR_ERR_WORKSPACE", 6: "GTR_ERR_RANGE"}

# every symbol include/gtr.h declares
EXPORTED = ("gtr_gla_fwd", "gtr_gla_fwd_f16", "gtr_gla_fwd_bf16", "gtr_gla_fwd_f32",
            "gtr_gla_workspace_bytes", "gtr_gla_fwd_ex", "gtr_gla_fwd_host",
            "gtr_gla_read_error", "gtr_gla_plan", "gtr_gla_workspace_init", "gtr_status_string",
            "gtr_version", "gtr_gla_fwd_noalloc", "gtr_gla_block_fwd", "gtr_sswiglu_dwconv",
            "gtr_gla_workspace_debug")


class GTRError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}" if what else STATUS.get(status, str(status)))


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libgtr.so not found at {LIB_PATH}; build it with "
            "`python gated_token_recurrence_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    fwd_args = [vp] * 5 + [i] * 7
    lib.gtr_gla_fwd.argtypes = fwd_args + [i, i, vp]
    for name in ("gtr_gla_fwd_f16", "gtr_gla_fwd_bf16", "gtr_gla_fwd_f32"):
        getattr(lib, name).argtypes = fwd_args + [vp]
    lib.gtr_gla_fwd_ex.argtypes = fwd_args + [i, i, i, vp, sz, vp]
    lib.gtr_gla_fwd_host.argtypes = fwd_args + [i, i, vp]
    lib.gtr_gla_fwd_noalloc.argtypes = fwd_args + [i, i, vp]
    f = ctypes.c_float
    lib.gtr_gla_block_fwd.argtypes = [vp] * 7 + [i, f, vp, vp, f, vp] + [i] * 10 + [vp, sz, vp]
    lib.gtr_sswiglu_dwconv.argtypes = [vp] * 5 + [i] * 5 + [vp]
    lib.gtr_gla_workspace_debug.argtypes = [vp, i, ctypes.c_uint, vp]
    lib.gtr_gla_workspace_bytes.argtypes = [i] * 8
    lib.gtr_gla_workspace_bytes.restype = sz
    lib.gtr_gla_read_error.argtypes = [vp, vp]
    lib.gtr_gla_workspace_init.argtypes = [vp, sz, vp]
    lib.gtr_gla_plan.argtypes = [i] * 7 + [ctypes.POINTER(i), ctypes.POINTER(i)]
    lib.gtr_status_string.argtypes = [i]
    lib.gtr_status_string.restype = ctypes.c_char_p
    lib.gtr_version.argtypes = []
    for name in ("gtr_gla_fwd", "gtr_gla_fwd_f16", "gtr_gla_fwd_bf16", "gtr_gla_fwd_f32",
                 "gtr_gla_fwd_ex", "gtr_gla_fwd_host", "gtr_gla_read_error", "gtr_gla_plan",
                 "gtr_gla_workspace_init", "gtr_version", "gtr_gla_fwd_noalloc", "gtr_gla_block_fwd",
                 "gtr_sswiglu_dwconv", "gtr_gla_workspace_debug"):
        getattr(lib, name).restype = ctypes.c_int
    return lib


lib = _load()


def _dtype_code(t) -> int:
    import torch
    return {torch.float32: F32, torch.float16: F16, torch.bfloat16: BF16}[t.dtype]


def default_out_dtype(in_dtype):
    """fp16 -> fp16, bf16 -> fp32, fp32 -> fp32."""
    import torch
    return torch.float16 if in_dtype == torch.float16 else torch.float32


def _check(st: int, what: str):
    if st != 0:
        raise GTRError(st, what)


def _stream_handle(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _shape(q, v, grid):
    B, L, heads, d_k = q.shape
    H, W = grid
    if H * W != L:
        raise ValueError(f"grid {H}x{W} does not match L={L}")
    return B, heads, H, W, d_k, v.shape[-1]


def workspace_bytes(B: int, heads: int, H: int, W: int, d_k: int = 64, d_v: int = 64,
                    in_dtype: int = F16, path: str = "auto") -> int:
    return int(lib.gtr_gla_workspace_bytes(B, heads, H, W, d_k, d_v, in_dtype, PATHS[path]))


def new_workspace(B: int, heads: int, H: int, W: int, d_k: int = 64, d_v: int = 64,
                  in_dtype: int = F16, path: str = "auto", device=None):
    """A zeroed uint8 CUDA tensor sized for :func:`gla_fwd` with ``workspace=``."""
    import torch
    n = max(256, workspace_bytes(B, heads, H, W, d_k, d_v, in_dtype, path))
    return torch.zeros(n, dtype=torch.uint8, device=device)


def gla_fwd(q, k, v, log_gamma, grid: Tuple[int, int], direction: int = L2R, out=None,
            path: str = "auto", workspace=None, stream=None):
    """Forward pass on CUDA tensors; returns ``out`` ([B, L, heads, d_v]).

    ``workspace`` (a uint8 CUDA tensor of at least :func:`workspace_bytes`,
    zeroed before its first use - see :func:`new_workspace`) selects the
    caller-managed-workspace entry (no allocation, capturable);
    without it the library's cached per-device workspace is used, and ``path``
    must then be "auto".
    """
    import torch
    B, heads, H, W, d_k, d_v = _shape(q, v, grid)
    if out is None:
        out = torch.empty((B, H * W, heads, d_v), dtype=default_out_dtype(q.dtype), device=q.device)
    for t in (q, k, v, log_gamma, out):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("gla_fwd takes contiguous CUDA tensors")
    if log_gamma.dtype != torch.float32:
        raise ValueError("log_gamma must be float32")
    if not (q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must share a dtype")
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), log_gamma.data_ptr(), out.data_ptr(),
            B, heads, H, W, d_k, d_v, int(direction), _dtype_code(q), _dtype_code(out))
    s = _stream_handle(stream)
    if workspace is None and path == "auto":
        _check(lib.gtr_gla_fwd(*args, s), "gtr_gla_fwd")
    else:
        if workspace is None:
            workspace = new_workspace(B, heads, H, W, d_k, d_v, _dtype_code(q), path, q.device)
        _check(lib.gtr_gla_fwd_ex(*args, PATHS[path], workspace.data_ptr(), workspace.numel(), s),
               "gtr_gla_fwd_ex")
    return out


def gla_block_fwd(q, k, v, grid: Tuple[int, int], direction: int = L2R, log_gamma=None,
                  gate_z=None, gate_w2=None, gate_b=None, gate_tau: float = 16.0,
                  out_gate=None, norm_w=None, norm_eps: float = 1e-6, out=None, path: str = "auto",
                  workspace=None, stream=None):
    """The GLA token mixer of a GTR block (``gtr_gla_block_fwd``) on CUDA tensors.

    Gates: either ``log_gamma`` [B, L, heads, d_k] fp32, or the low-rank producer
    ``gate_z`` [B, L, r] fp32 with ``gate_w2`` [r, heads*d_k] and ``gate_b`` [heads*d_k]
    (log gamma = logsigmoid(z W2 + b) / gate_tau).  With ``out_gate`` [B, L, heads, d_v]
    (input dtype) and ``norm_w`` [d_v] fp32 the output is RMSNorm(o) * norm_w * SiLU(out_gate).
    """
    import torch
    B, heads, H, W, d_k, d_v = _shape(q, v, grid)
    if out is None:
        out = torch.empty((B, H * W, heads, d_v), dtype=default_out_dtype(q.dtype), device=q.device)
    tensors = [t for t in (q, k, v, log_gamma, gate_z, gate_w2, gate_b, out_gate, norm_w, out) if t is not None]
    for t in tensors:
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("gla_block_fwd takes contiguous CUDA tensors")
    for t in (log_gamma, gate_z, gate_w2, gate_b, norm_w):
        if t is not None and t.dtype != torch.float32:
            raise ValueError("gates, gate factors and the norm weight are float32")
    ptr = lambda t: None if t is None else t.data_ptr()
    rank = 0 if gate_z is None else int(gate_z.shape[-1])
    ws, wsb = (None, 0) if workspace is None else (workspace.data_ptr(), workspace.numel())
    st = lib.gtr_gla_block_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), ptr(log_gamma), ptr(gate_z),
                               ptr(gate_w2), ptr(gate_b), rank, float(gate_tau), ptr(out_gate), ptr(norm_w),
                               float(norm_eps), out.data_ptr(), B, heads, H, W, d_k, d_v, int(direction),
                               _dtype_code(q), _dtype_code(out), PATHS[path], ws, wsb, _stream_handle(stream))
    _check(st, "gtr_gla_block_fwd")
    return out


def sswiglu_dwconv(xg, xv, conv_w, conv_b, grid: Tuple[int, int], out=None, stream=None):
    """SiLU(xg) * DWConv3x3(xv) on CUDA tensors ([B, L, C], L = H * W; conv_w [C, 3, 3] fp32,
    conv_b [C] fp32 or None) through ``gtr_sswiglu_dwconv``."""
    import torch
    B, L, C = xv.shape
    H, W = grid
    if H * W != L or xg.shape != xv.shape or xg.dtype != xv.dtype:
        raise ValueError("xg and xv must both be [B, H*W, C] of one dtype")
    if out is None:
        out = torch.empty_like(xv)
    for t in (xg, xv, conv_w, out) + (() if conv_b is None else (conv_b,)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("sswiglu_dwconv takes contiguous CUDA tensors")
    st = lib.gtr_sswiglu_dwconv(xg.data_ptr(), xv.data_ptr(), conv_w.data_ptr(),
                                None if conv_b is None else conv_b.data_ptr(), out.data_ptr(), B, H, W, C,
                                _dtype_code(xv), _stream_handle(stream))
    _check(st, "gtr_sswiglu_dwconv")
    return out


def gla_fwd_host(q, k, v, log_gamma, out, grid: Tuple[int, int], direction: int = L2R,
                 stream=None):
    """Forward pass on HOST (CPU, ideally pinned) tensors through ``gtr_gla_fwd_host``.

    The library copies the inputs in, runs, copies ``out`` back and synchronises.
    """
    B, heads, H, W, d_k, d_v = _shape(q, v, grid)
    for t in (q, k, v, log_gamma, out):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("gla_fwd_host takes contiguous CPU tensors")
    st = lib.gtr_gla_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), log_gamma.data_ptr(),
                              out.data_ptr(), B, heads, H, W, d_k, d_v, int(direction),
                              _dtype_code(q), _dtype_code(out), _stream_handle(stream))
    _check(st, "gtr_gla_fwd_host")
    return out


def plan(B: int, heads: int, H: int, W: int, d_k: int = 64, d_v: int = 64,
         in_dtype: int = F16) -> Tuple[str, int]:
    """(path name, kernel launches per call) that the dispatcher picks for this problem."""
    path, launches = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib.gtr_gla_plan(B, heads, H, W, d_k, d_v, in_dtype, ctypes.byref(path),
                            ctypes.byref(launches)), "gtr_gla_plan")
    name = {v: k for k, v in PATHS.items()}[path.value]
    return name, launches.value


def read_error(workspace=None, stream=None) -> int:
    """Synchronise and return (and clear) the device error word; 0 = none."""
    ptr = None if workspace is None else workspace.data_ptr()
    return int(lib.gtr_gla_read_error(ptr, _stream_handle(stream)))


def status_string(st: int) -> str:
    return lib.gtr_status_string(int(st)).decode()


def version() -> int:
    return int(lib.gtr_version())
