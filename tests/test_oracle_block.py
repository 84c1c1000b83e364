"""Pins for the oracle's GTR block pieces: the low-rank gate producer, the RMSNorm +
SiLU output-gate epilogue and the Spatial SwiGLU depthwise 3x3 stencil.

Each function is checked against library routines (scipy, torch CPU in float64),
hand-worked values and special cases with closed forms, so that a dropped term, a
transposed operand, a wrong sign, a misplaced head slice or a flipped convolution
orientation fails at least one check.  CPU only.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

import oracle


# ---------------------------------------------------------------- low-rank gate producer
def test_lowrank_gate_hand_worked_values():
    """z W2 + b chosen to hit 0, ln 3 and -ln 3, where log sigmoid is -ln 2, ln(3/4) and
    ln(1/4); tau = 16; one token, one head of d_k = 3, rank 2."""
    ln3 = math.log(3.0)
    z = np.array([[[1.0, 2.0]]])                 # [B=1, L=1, r=2]
    w2 = np.array([[0.0, ln3, 0.0],              # [r=2, heads*d_k=3]
                   [0.0, 0.0, -ln3 / 2.0]])
    b = np.array([0.0, 0.0, 0.0])
    lg = oracle.lowrank_log_gamma(z, w2, b, 16.0, heads=1, d_k=3)
    np.testing.assert_allclose(lg[0, 0, 0], np.array([-math.log(2.0), math.log(0.75), math.log(0.25)]) / 16.0,
                               rtol=1e-14, atol=0)


def test_lowrank_gate_against_library_log_expit_and_head_slices():
    rng = np.random.default_rng(5)
    B, L, r, heads, dk = 2, 7, 16, 3, 8
    z = rng.standard_normal((B, L, r))
    w2 = rng.standard_normal((r, heads * dk))
    b = rng.standard_normal(heads * dk)
    lg = oracle.lowrank_log_gamma(z, w2, b, 16.0, heads, dk)
    ref = scipy.special.log_expit(np.einsum("blr,rc->blc", z, w2) + b) / 16.0
    np.testing.assert_allclose(lg, ref.reshape(B, L, heads, dk), rtol=1e-13, atol=1e-15)
    # gamma^tau = sigmoid(z W2 + b)
    np.testing.assert_allclose(np.exp(16.0 * lg).reshape(B, L, heads * dk),
                               scipy.special.expit(np.einsum("blr,rc->blc", z, w2) + b), rtol=1e-13)
    # head h's gates depend on columns h*dk .. h*dk+dk-1 of W2 only
    w2b = w2.copy()
    w2b[:, dk:2 * dk] += 1.0
    lg2 = oracle.lowrank_log_gamma(z, w2b, b, 16.0, heads, dk)
    assert np.array_equal(lg2[:, :, 0], lg[:, :, 0]) and np.array_equal(lg2[:, :, 2], lg[:, :, 2])
    assert not np.allclose(lg2[:, :, 1], lg[:, :, 1])


def test_lowrank_gate_limits():
    """Large positive pre-activations keep everything (log gamma -> -exp(-g)/tau), large
    negative ones give log gamma -> g / tau; neither overflows."""
    z = np.array([[[1.0]]])
    for g, expect in ((60.0, -math.exp(-60.0) / 4.0), (-700.0, -700.0 / 4.0), (-40.0, (-40.0 - math.exp(-40.0)) / 4.0)):
        lg = oracle.lowrank_log_gamma(z, np.array([[g]]), np.array([0.0]), 4.0, 1, 1)
        assert np.isfinite(lg).all()
        np.testing.assert_allclose(lg[0, 0, 0, 0], expect, rtol=1e-12)


def test_lowrank_recurrence_with_unit_gates_is_causal_linear_attention():
    """W2 = 0 and a large bias: gamma = 1 to double precision, so the block is textbook causal
    linear attention, o_t = d_k^-1/2 q_t sum_{s<=t} k_s^T v_s (prefix sums, written here
    without the recurrence)."""
    rng = np.random.default_rng(9)
    B, H, W, heads, dk, dv, r = 1, 4, 6, 2, 8, 5, 16
    L = H * W
    q = rng.standard_normal((B, L, heads, dk))
    k = rng.standard_normal((B, L, heads, dk))
    v = rng.standard_normal((B, L, heads, dv))
    z = rng.standard_normal((B, L, r))
    out = oracle.gla_fwd_lowrank(q, k, v, z, np.zeros((r, heads * dk)), np.full(heads * dk, 80.0), 16.0, H, W, 2)
    order = oracle.scan_order(2, H, W)
    kv = np.einsum("blhk,blhv->blhkv", k[:, order], v[:, order]).cumsum(axis=1)
    ref = np.empty_like(out)
    ref[:, order] = np.einsum("blhk,blhkv->blhv", q[:, order], kv) / math.sqrt(dk)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- RMSNorm + SiLU output gate
def test_gate_epilogue_hand_worked_values():
    """o = (3, 4): rms = sqrt(12.5); gate (0, ln 3): SiLU = 0 and ln 3 * 3/4; weight (2, 0.5)."""
    o = np.array([[[[3.0, 4.0]]]])
    r = np.array([[[[0.0, math.log(3.0)]]]])
    w = np.array([2.0, 0.5])
    y = oracle.rmsnorm_silu_gate(o, r, w, 0.0)
    rms = math.sqrt(12.5)
    np.testing.assert_allclose(y[0, 0, 0], [0.0, 4.0 / rms * 0.5 * math.log(3.0) * 0.75], rtol=1e-14, atol=0)


def test_gate_epilogue_against_torch_library():
    rng = np.random.default_rng(3)
    o = rng.standard_normal((2, 9, 3, 64)) * 5.0
    r = rng.standard_normal((2, 9, 3, 64))
    w = 1.0 + 0.1 * rng.standard_normal(64)
    for eps in (0.0, 1e-6, 1e-2):
        y = oracle.rmsnorm_silu_gate(o, r, w, eps)
        ref = F.rms_norm(torch.from_numpy(o), (64,), torch.from_numpy(w), eps) * F.silu(torch.from_numpy(r))
        np.testing.assert_allclose(y, ref.numpy(), rtol=1e-12, atol=1e-13)


def test_gate_epilogue_is_scale_invariant_and_per_row():
    rng = np.random.default_rng(4)
    o = rng.standard_normal((1, 5, 2, 16))
    r = rng.standard_normal((1, 5, 2, 16))
    w = rng.standard_normal(16)
    y = oracle.rmsnorm_silu_gate(o, r, w, 0.0)
    np.testing.assert_allclose(oracle.rmsnorm_silu_gate(1e-7 * o, r, w, 0.0), y, rtol=1e-12)
    o2 = o.copy()
    o2[0, 3, 1] *= 10.0  # one token-head row: only that row's norm changes
    y2 = oracle.rmsnorm_silu_gate(o2, r, w, 0.0)
    mask = np.ones(o.shape[:3], dtype=bool)
    mask[0, 3, 1] = False
    np.testing.assert_array_equal(y2[mask], y[mask])
    np.testing.assert_allclose(y2[0, 3, 1], y[0, 3, 1], rtol=1e-12)  # (scale invariance again)


def test_gated_recurrence_composes_the_two_oracles():
    rng = np.random.default_rng(6)
    q, k, v = (rng.standard_normal((1, 12, 2, 8)) for _ in range(3))
    lg = -0.2 * rng.random((1, 12, 2, 8))
    r = rng.standard_normal((1, 12, 2, 8))
    w = rng.standard_normal(8)
    o = oracle.gla_fwd_bruteforce(q, k, v, lg, 3, 4, 1)
    ref = F.rms_norm(torch.from_numpy(o), (8,), torch.from_numpy(w), 1e-6) * F.silu(torch.from_numpy(r))
    np.testing.assert_allclose(oracle.gla_fwd_gated(q, k, v, lg, r, w, 1e-6, 3, 4, 1), ref.numpy(), rtol=1e-10)


# ---------------------------------------------------------------- Spatial SwiGLU stencil
def _torch_dwconv(xv, w, b, H, W):
    B, L, C = xv.shape
    x = torch.from_numpy(xv).reshape(B, H, W, C).permute(0, 3, 1, 2)
    out = F.conv2d(x, torch.from_numpy(w).reshape(C, 1, 3, 3), None if b is None else torch.from_numpy(b),
                   padding=1, groups=C)
    return out.permute(0, 2, 3, 1).reshape(B, L, C).numpy()


@pytest.mark.parametrize("bias", [True, False])
def test_stencil_against_torch_conv2d(bias):
    rng = np.random.default_rng(7)
    B, H, W, C = 2, 5, 7, 6
    xg = rng.standard_normal((B, H * W, C))
    xv = rng.standard_normal((B, H * W, C))
    w = rng.standard_normal((C, 3, 3))
    b = rng.standard_normal(C) if bias else None
    z = oracle.sswiglu_dwconv(xg, xv, w, b, H, W)
    ref = F.silu(torch.from_numpy(xg)).numpy() * _torch_dwconv(xv, w, b, H, W)
    np.testing.assert_allclose(z, ref, rtol=1e-12, atol=1e-13)


def test_stencil_special_kernels():
    """Delta kernel: the identity; all-ones kernel on a constant image: the count of
    in-grid neighbours (9 inside, 6 on edges, 4 at corners); kernel tap (dy, dx) = (0, 1):
    each token takes the value of the token one row above (zero on the first row)."""
    B, H, W, C = 1, 4, 5, 3
    rng = np.random.default_rng(8)
    xg = rng.standard_normal((B, H * W, C))
    silu = xg / (1.0 + np.exp(-xg))
    xv = rng.standard_normal((B, H * W, C))
    delta = np.zeros((C, 3, 3))
    delta[:, 1, 1] = 1.0
    np.testing.assert_allclose(oracle.sswiglu_dwconv(xg, xv, delta, None, H, W), silu * xv, rtol=1e-15)
    ones = np.ones((C, 3, 3))
    cnt = oracle.sswiglu_dwconv(np.full((B, H * W, C), 40.0), np.ones((B, H * W, C)), ones, None, H, W)
    cnt = cnt[0, :, 0].reshape(H, W) / 40.0
    expect = np.full((H, W), 9.0)
    expect[0, :] = expect[-1, :] = 6.0
    expect[:, 0] = expect[:, -1] = 6.0
    expect[0, 0] = expect[0, -1] = expect[-1, 0] = expect[-1, -1] = 4.0
    np.testing.assert_allclose(cnt, expect, rtol=1e-12)
    up = np.zeros((C, 3, 3))
    up[:, 0, 1] = 1.0
    z = oracle.sswiglu_dwconv(xg, xv, up, None, H, W).reshape(B, H, W, C)
    shifted = np.zeros((B, H, W, C))
    shifted[:, 1:] = xv.reshape(B, H, W, C)[:, :-1]
    np.testing.assert_allclose(z, silu.reshape(B, H, W, C) * shifted, rtol=1e-15)


# ---------------------------------------------------------------- the pins catch plausible slips
def _mut_gate(kind):
    def f(z, w2, b, tau, heads, dk):
        B, L, _ = z.shape
        if kind == "no_tau":
            g = z @ w2 + b
            return oracle._log_sigmoid(g).reshape(B, L, heads, dk)
        if kind == "sigmoid_not_log":
            return (scipy.special.expit(z @ w2 + b) / tau).reshape(B, L, heads, dk)
        if kind == "head_major_columns":  # columns read as [d_k][heads]
            g = (z @ w2 + b).reshape(B, L, dk, heads).transpose(0, 1, 3, 2)
            return oracle._log_sigmoid(g) / tau
        raise ValueError(kind)
    return f


def _mut_epilogue(kind):
    def f(o, r, w, eps):
        if kind == "sum_not_mean":
            return o / np.sqrt(np.sum(o * o, axis=-1, keepdims=True) + eps) * w * r / (1 + np.exp(-r))
        if kind == "sigmoid_gate":
            return o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps) * w / (1 + np.exp(-r))
        if kind == "norm_over_heads":
            return o / np.sqrt(np.mean(o * o, axis=(-2, -1), keepdims=True) + eps) * w * r / (1 + np.exp(-r))
        raise ValueError(kind)
    return f


def _mut_stencil(kind):
    def f(xg, xv, w, b, H, W):
        if kind == "flipped_kernel":  # a true convolution instead of the layer's correlation
            return oracle.sswiglu_dwconv(xg, xv, w[:, ::-1, ::-1].copy(), b, H, W)
        if kind == "transposed_grid":
            B, L, C = xv.shape
            t = lambda a: a.reshape(B, H, W, C).transpose(0, 2, 1, 3).reshape(B, L, C)
            return t(oracle.sswiglu_dwconv(t(xg), t(xv), w.transpose(0, 2, 1).copy(), b, W, H))
        if kind == "wrapped_border":
            B, L, C = xv.shape
            img = xv.reshape(B, H, W, C)
            conv = sum(np.roll(img, (1 - dy, 1 - dx), axis=(1, 2)) * w[:, dy, dx] for dy in range(3) for dx in range(3))
            return xg / (1 + np.exp(-xg)) * (conv.reshape(B, L, C) + (0 if b is None else b))
        raise ValueError(kind)
    return f


@pytest.mark.parametrize("kind", ["no_tau", "sigmoid_not_log", "head_major_columns"])
def test_gate_pins_reject_planted_mistakes(kind):
    rng = np.random.default_rng(5)
    B, L, r, heads, dk = 2, 7, 16, 3, 8
    z, w2, b = rng.standard_normal((B, L, r)), rng.standard_normal((r, heads * dk)), rng.standard_normal(heads * dk)
    ref = (scipy.special.log_expit(z @ w2 + b) / 16.0).reshape(B, L, heads, dk)
    assert np.allclose(oracle.lowrank_log_gamma(z, w2, b, 16.0, heads, dk), ref, rtol=1e-12)
    assert not np.allclose(_mut_gate(kind)(z, w2, b, 16.0, heads, dk), ref, rtol=1e-6)


@pytest.mark.parametrize("kind", ["sum_not_mean", "sigmoid_gate", "norm_over_heads"])
def test_epilogue_pins_reject_planted_mistakes(kind):
    rng = np.random.default_rng(3)
    o, r = rng.standard_normal((2, 9, 3, 64)), rng.standard_normal((2, 9, 3, 64))
    w = 1.0 + 0.1 * rng.standard_normal(64)
    ref = (F.rms_norm(torch.from_numpy(o), (64,), torch.from_numpy(w), 1e-6) * F.silu(torch.from_numpy(r))).numpy()
    assert np.allclose(oracle.rmsnorm_silu_gate(o, r, w, 1e-6), ref, rtol=1e-12)
    assert not np.allclose(_mut_epilogue(kind)(o, r, w, 1e-6), ref, rtol=1e-6)


@pytest.mark.parametrize("kind", ["flipped_kernel", "transposed_grid", "wrapped_border"])
def test_stencil_pins_reject_planted_mistakes(kind):
    rng = np.random.default_rng(7)
    B, H, W, C = 2, 5, 7, 6
    xg, xv = rng.standard_normal((B, H * W, C)), rng.standard_normal((B, H * W, C))
    w, b = rng.standard_normal((C, 3, 3)), rng.standard_normal(C)
    ref = F.silu(torch.from_numpy(xg)).numpy() * _torch_dwconv(xv, w, b, H, W)
    assert np.allclose(oracle.sswiglu_dwconv(xg, xv, w, b, H, W), ref, rtol=1e-12)
    assert not np.allclose(_mut_stencil(kind)(xg, xv, w, b, H, W), ref, rtol=1e-6)
