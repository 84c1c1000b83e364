"""Oracle for the key-only gated linear attention forward pass.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA path and never imports it.

Three independent readings of the same operation, all in IEEE double:

* :func:`gla_fwd` - the plain sequential recurrence (C, ``gtr_oracle.c``)
  ``S_t = Diag(gamma_t) S_{t-1} + k_t^T v_t``, ``o_t = d_k^{-1/2} q_t S_t``
  (GTR digest page paper.rainbus.top, prerequisite "Gated linear attention";
  0539edu.com section 3.1).  This is THE oracle.
* :func:`gla_fwd_bruteforce` - the closed form of that recurrence,
  ``o_t = d_k^{-1/2} sum_{s<=t} (q_t * prod_{r=s+1..t} gamma_r) . k_s  v_s``,
  written with explicit products (tiny inputs only).
* :func:`gla_fwd_chunked` - the chunkwise form from the same digest page
  (prerequisite "Chunkwise parallel"; step 5 of "Method details"): per chunk a
  summary ``U_c`` and decay ``d_c``, boundary states
  ``S_[c+1] = Diag(d_c) S_[c] + U_c``, and per-chunk outputs.  It reaches the
  sequential result up to rounding for any chunk length C.

Inputs of any float dtype are upcast exactly to float64 before use.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gtr_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libgtr_oracle.so")
_lib = None

DIRECTIONS = {"l2r": 0, "r2l": 1, "t2b": 2, "b2t": 3}


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (OpenMP when available).  Returns the .so path."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    base = ["gcc", "-O2", "-fPIC", "-shared", "-std=c99", "-o", tmp, _SRC, "-lm"]
    try:
        subprocess.run(base[:1] + ["-fopenmp"] + base[1:], check=True,
                       capture_output=True)
    except subprocess.CalledProcessError:
        subprocess.run(base, check=True, capture_output=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        lib.gtr_oracle_fwd.argtypes = [dp, dp, dp, dp, dp] + [ctypes.c_int] * 8
        lib.gtr_oracle_fwd.restype = ctypes.c_int
        lib.gtr_oracle_scan_token.argtypes = [ctypes.c_long, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int]
        lib.gtr_oracle_scan_token.restype = ctypes.c_long
        lib.gtr_oracle_max_threads.argtypes = []
        lib.gtr_oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    """Threads the C oracle uses when not told otherwise."""
    return int(_load().gtr_oracle_max_threads())


def _f64(x) -> np.ndarray:
    """Exact upcast of a numpy array or (CPU/GPU) torch tensor to C-contiguous float64."""
    if hasattr(x, "detach"):  # torch tensor, any float dtype: the cast to float64 is exact
        import torch
        x = x.detach().to(device="cpu", dtype=torch.float64).contiguous().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def scan_token(s: int, direction: int, H: int, W: int) -> int:
    """Token index m = y*W + x visited at scan position s (C oracle's reading)."""
    return int(_load().gtr_oracle_scan_token(s, direction, H, W))


def gla_fwd(q, k, v, log_gamma, H: int, W: int, direction: int = 0,
            threads: int = 0) -> np.ndarray:
    """Sequential recurrence in float64.  Tensors are [B, L, heads, d], L = H*W."""
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(log_gamma)
    B, L, heads, d_k = q.shape
    d_v = v.shape[-1]
    if L != H * W or k.shape != q.shape or g.shape != q.shape or v.shape[:3] != q.shape[:3]:
        raise ValueError("shape mismatch")
    out = np.empty((B, L, heads, d_v), dtype=np.float64)
    dp = ctypes.POINTER(ctypes.c_double)
    rc = _load().gtr_oracle_fwd(q.ctypes.data_as(dp), k.ctypes.data_as(dp),
                                v.ctypes.data_as(dp), g.ctypes.data_as(dp),
                                out.ctypes.data_as(dp), B, heads, H, W, d_k, d_v,
                                int(direction), int(threads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return out


def scan_order(direction: int, H: int, W: int) -> np.ndarray:
    """Token index for every scan position, as a numpy array (same reading as the C oracle).

    left->right: rows top to bottom, x ascending; right->left: rows top to
    bottom, x descending; top->bottom: columns left to right, y ascending;
    bottom->top: columns left to right, y descending.
    """
    y, x = np.meshgrid(np.arange(H), np.arange(W), indexing="ij")
    if direction == 0:
        return (y * W + x).reshape(-1)
    if direction == 1:
        return (y * W + (W - 1 - x)).reshape(-1)
    if direction == 2:
        return (y * W + x).T.reshape(-1)
    if direction == 3:
        return ((H - 1 - y) * W + x).T.reshape(-1)
    raise ValueError("direction must be 0..3")


def gla_fwd_bruteforce(q, k, v, log_gamma, H: int, W: int, direction: int = 0) -> np.ndarray:
    """Closed form with explicit gate products; O(L^2) numpy calls, meant for L <= 64."""
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(log_gamma)
    B, L, heads, d_k = q.shape
    order = scan_order(direction, H, W)
    gam = np.exp(g)
    out = np.zeros(v.shape, dtype=np.float64)
    for b in range(B):
        for h in range(heads):
            for t in range(L):
                mt = order[t]
                acc = np.zeros(v.shape[-1])
                for s in range(t + 1):
                    ms = order[s]
                    decay = np.ones(d_k)
                    for r in range(s + 1, t + 1):
                        decay = decay * gam[b, order[r], h]
                    acc = acc + np.dot(q[b, mt, h] * decay, k[b, ms, h]) * v[b, ms, h]
                out[b, mt, h] = acc / np.sqrt(d_k)
    return out


def gla_fwd_chunked(q, k, v, log_gamma, H: int, W: int, direction: int = 0,
                    C: int = 64) -> np.ndarray:
    """Chunkwise form: chunk summaries, boundary-state scan, per-chunk outputs.

    Per chunk with in-chunk inclusive cumulative log-gates A (rows = positions):
      d_c    = exp(A[last])
      U_c    = (K * exp(A[last] - A))^T V
      o_i    = d_k^{-1/2} [ (q_i * exp(A_i)) S_[c]  +  sum_{j<=i} (q_i * exp(A_i - A_j)) . k_j  v_j ]
      S_[c+1] = Diag(d_c) S_[c] + U_c
    A trailing partial chunk is handled as a shorter chunk.
    """
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(log_gamma)
    B, L, heads, d_k = q.shape
    d_v = v.shape[-1]
    order = scan_order(direction, H, W)
    out = np.zeros((B, L, heads, d_v), dtype=np.float64)
    for b in range(B):
        for h in range(heads):
            Q, K, V, G = q[b, order, h], k[b, order, h], v[b, order, h], g[b, order, h]
            O = np.zeros((L, d_v))
            S = np.zeros((d_k, d_v))
            for c0 in range(0, L, C):
                sl = slice(c0, min(c0 + C, L))
                Qc, Kc, Vc = Q[sl], K[sl], V[sl]
                A = np.cumsum(G[sl], axis=0)
                n = A.shape[0]
                inter = (Qc * np.exp(A)) @ S
                # exp(A_i - A_j) for j <= i is a product of gates, so <= 1
                diff = A[:, None, :] - A[None, :, :]
                mask = np.tril(np.ones((n, n), dtype=bool))
                P = np.einsum("ik,jk,ijk->ij", Qc, Kc, np.exp(np.where(mask[:, :, None], diff, -np.inf)))
                O[sl] = (inter + P @ Vc) / np.sqrt(d_k)
                U = (Kc * np.exp(A[-1] - A)).T @ Vc
                S = np.exp(A[-1])[:, None] * S + U
            out[b, order, h] = O
    return out


# ----------------------------------------------------------------------------- GTR block pieces
def _log_sigmoid(g: np.ndarray) -> np.ndarray:
    """log(sigmoid(g)) = -log(1 + exp(-g)), written so that neither branch overflows."""
    return np.minimum(g, 0.0) - np.log1p(np.exp(-np.abs(g)))


def lowrank_log_gamma(z, w2, bias, tau: float, heads: int, d_k: int) -> np.ndarray:
    """The low-rank data-dependent retention gate of GTR, in log form.

    GTR digest page (paper.rainbus.top), section "Core method": the key-side gate is
    gamma_t = sigmoid(x_t W1 W2 + b)^(1/tau) with a rank-16 factorisation and tau = 16.
    With z = x W1 (the rank-r projection of each token, [B, L, r]), W2 of shape
    [r, heads * d_k] and b of shape [heads * d_k]:

        log gamma[b, m, h, :] = log sigmoid(z[b, m] W2 + b)[h * d_k : (h + 1) * d_k] / tau

    Returns [B, L, heads, d_k] in float64.
    """
    z, w2, bias = _f64(z), _f64(w2), _f64(bias)
    B, L, _ = z.shape
    g = z @ w2 + bias
    return (_log_sigmoid(g) / float(tau)).reshape(B, L, heads, d_k)


def gla_fwd_lowrank(q, k, v, z, w2, bias, tau: float, H: int, W: int, direction: int = 0) -> np.ndarray:
    """The recurrence (:func:`gla_fwd`) with its gates produced by :func:`lowrank_log_gamma`."""
    qq = _f64(q)
    heads, d_k = qq.shape[2], qq.shape[3]
    return gla_fwd(qq, k, v, lowrank_log_gamma(z, w2, bias, tau, heads, d_k), H, W, direction)


def rmsnorm_silu_gate(o, gate, weight, eps: float) -> np.ndarray:
    """The GLA output epilogue: RMSNorm over the d_v channels of each token-head, the norm
    weight, then the SiLU-activated output gate.

    0539edu.com, appendix E.3.1: the end-to-end implementation fuses RMSNorm and a
    SiLU-activated output gate into the GLA kernel's output epilogue.  Per token-head row
    o (d_v values), gate r (d_v values) and weight w (d_v values, shared by the heads):

        y_j = o_j / sqrt(mean_i o_i^2 + eps) * w_j * r_j * sigmoid(r_j)
    """
    o, r, w = _f64(o), _f64(gate), _f64(weight)
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + float(eps))
    return o / rms * w * (r / (1.0 + np.exp(-r)))


def gla_fwd_gated(q, k, v, log_gamma, gate, weight, eps: float, H: int, W: int,
                  direction: int = 0) -> np.ndarray:
    """The recurrence (:func:`gla_fwd`) followed by :func:`rmsnorm_silu_gate`."""
    return rmsnorm_silu_gate(gla_fwd(q, k, v, log_gamma, H, W, direction), gate, weight, eps)


def sswiglu_dwconv(xg, xv, conv_w, conv_b, H: int, W: int) -> np.ndarray:
    """The spatial part of GTR's Spatial SwiGLU: SiLU(X W_g) * DWConv3x3(X W_v).

    GTR digest page, prerequisite "SwiGLU" and section "Core method": the channel mixer is
    Y = SiLU(X W_g) (.) DWConv3x3(X W_v) W_o, a 3x3 depthwise convolution in the value
    branch that mixes neighbouring patches (0539edu.com section 3.1 "Spatial SwiGLU").
    This computes the product before W_o from the two projections xg = X W_g and
    xv = X W_v, both [B, L, C] with token m = y * W + x on the H x W grid.  The
    convolution is channel by channel, stride 1, zero padding 1, in the cross-correlation
    convention of a convolution layer:

        conv[b, y, x, c] = bias[c] + sum_{dy, dx in 0..2} w[c, dy, dx] * xv[b, y+dy-1, x+dx-1, c]

    conv_b may be None (no bias).  Returns [B, L, C] in float64.
    """
    xg, xv, w = _f64(xg), _f64(xv), _f64(conv_w)
    B, L, C = xv.shape
    if L != H * W or xg.shape != xv.shape or w.shape != (C, 3, 3):
        raise ValueError("shape mismatch")
    img = np.zeros((B, H + 2, W + 2, C))
    img[:, 1:H + 1, 1:W + 1, :] = xv.reshape(B, H, W, C)
    conv = np.zeros((B, H, W, C))
    for dy in range(3):
        for dx in range(3):
            conv += img[:, dy:dy + H, dx:dx + W, :] * w[:, dy, dx]
    if conv_b is not None:
        conv += _f64(conv_b)
    silu = xg / (1.0 + np.exp(-xg))
    return silu * conv.reshape(B, L, C)
