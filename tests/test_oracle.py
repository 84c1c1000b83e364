"""Pins for the oracle: it is checked against things other than itself.

Every check here runs on the CPU.  The pins are chosen so that a plausible
slip in the oracle (a dropped term, a sign, an index off by one, a decay on
the wrong side, the wrong scale, a wrong scan order) fails at least one of
them; ``test_pins_reject_planted_mistakes`` demonstrates that on purpose-built
wrong variants.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from gtr_inputs import WORKLOADS, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_case(B, L, heads, dk, dv, seed, gate_scale=0.3):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, L, heads, dk))
    k = rng.standard_normal((B, L, heads, dk))
    v = rng.standard_normal((B, L, heads, dv))
    lg = -gate_scale * rng.random((B, L, heads, dk))  # log gamma in (-gate_scale, 0]
    return q, k, v, lg


# ---------------------------------------------------------------- worked example
def test_hand_worked_example():
    """Three tokens, d_k=2, d_v=1, gamma=(1/2, 1/4), q=(1,1); values worked by hand.

    S_0 = [2, 0]^T                       -> o_0 = 2 / sqrt(2)
    S_1 = Diag(1/2,1/4) S_0 + [0, 3]^T = [1, 3]^T      -> o_1 = 4 / sqrt(2)
    S_2 = Diag(1/2,1/4) S_1 + [5, 5]^T = [5.5, 5.75]^T -> o_2 = 11.25 / sqrt(2)
    """
    q = np.ones((1, 3, 1, 2))
    k = np.array([[1, 0], [0, 1], [1, 1]], dtype=float).reshape(1, 3, 1, 2)
    v = np.array([2, 3, 5], dtype=float).reshape(1, 3, 1, 1)
    lg = np.log(np.tile(np.array([0.5, 0.25]), (1, 3, 1, 1)))
    out = oracle.gla_fwd(q, k, v, lg, H=1, W=3, direction=0)
    expect = np.array([2.0, 4.0, 11.25]) / math.sqrt(2.0)
    np.testing.assert_allclose(out[0, :, 0, 0], expect, rtol=1e-15, atol=0)


def test_geometric_closed_form():
    """q=k=1, constant per-channel gate g_k: o_t[j] = v_j/sqrt(dk) * sum_k (1-g_k^(t+1))/(1-g_k)."""
    L, dk, dv = 50, 3, 2
    gk = np.array([0.9, 0.5, 0.99])
    vj = np.array([1.5, -2.0])
    q = np.ones((1, L, 1, dk))
    k = np.ones((1, L, 1, dk))
    v = np.tile(vj, (1, L, 1, 1))
    lg = np.tile(np.log(gk), (1, L, 1, 1))
    out = oracle.gla_fwd(q, k, v, lg, H=5, W=10, direction=0)
    t = np.arange(L)[:, None]
    geo = ((1 - gk[None, :] ** (t + 1)) / (1 - gk[None, :])).sum(axis=1)
    expect = geo[:, None] * vj[None, :] / math.sqrt(dk)
    np.testing.assert_allclose(out[0, :, 0, :], expect, rtol=1e-13)


# ---------------------------------------------------------------- closed forms
@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_bruteforce_quadratic_form(direction):
    """Sequential recurrence == explicit sum over s <= t with gate products (d_k != d_v)."""
    H, W = 3, 4
    q, k, v, lg = rand_case(2, H * W, 2, 5, 3, seed=10 + direction)
    a = oracle.gla_fwd(q, k, v, lg, H, W, direction)
    b = oracle.gla_fwd_bruteforce(q, k, v, lg, H, W, direction)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def test_gamma_one_is_causal_linear_attention():
    """log gamma = 0: o_t = d_k^{-1/2} q_t sum_{s<=t} k_s^T v_s (textbook causal linear attention)."""
    H, W, dk, dv = 6, 7, 4, 6
    q, k, v, _ = rand_case(1, H * W, 3, dk, dv, seed=3)
    lg = np.zeros_like(q)
    out = oracle.gla_fwd(q, k, v, lg, H, W, 0)
    kv = np.einsum("blhk,blhj->blhkj", k, v)
    S = np.cumsum(kv, axis=1)
    expect = np.einsum("blhk,blhkj->blhj", q, S) / math.sqrt(dk)
    np.testing.assert_allclose(out, expect, rtol=1e-12, atol=1e-12)


def test_gamma_zero_keeps_only_current_token():
    """log gamma = -1e4 (gamma underflows to 0): o_t = d_k^{-1/2} (q_t . k_t) v_t."""
    H, W, dk, dv = 4, 5, 6, 3
    q, k, v, _ = rand_case(2, H * W, 2, dk, dv, seed=4)
    lg = np.full_like(q, -1e4)
    for direction in range(4):
        out = oracle.gla_fwd(q, k, v, lg, H, W, direction)
        expect = np.einsum("blhk,blhk->blh", q, k)[..., None] * v / math.sqrt(dk)
        np.testing.assert_allclose(out, expect, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("C", [1, 7, 16, 64, 256])
def test_chunked_equals_sequential(C):
    """The chunkwise form reaches the sequential result for any chunk length (incl. a ragged tail)."""
    H, W = 16, 16
    q, k, v, lg = rand_case(1, H * W, 2, 8, 5, seed=5, gate_scale=0.2)
    for direction in (0, 2):
        a = oracle.gla_fwd(q, k, v, lg, H, W, direction)
        b = oracle.gla_fwd_chunked(q, k, v, lg, H, W, direction, C=C)
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-10)


def test_chunked_equals_sequential_on_tiny_workload():
    w = WORKLOADS["tiny"]
    q, k, v, lg = make_inputs(w, w.seed(0))
    a = oracle.gla_fwd(q, k, v, lg, w.H, w.W, 0)
    b = oracle.gla_fwd_chunked(q, k, v, lg, w.H, w.W, 0, C=64)
    np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-10)


# ---------------------------------------------------------------- scan orders
def test_scan_orders_on_2x3_grid():
    """Grid y in {0,1}, x in {0,1,2}; token m = 3y + x.  v_m = 2^m, q = k = 1, gamma = 1, so
    o at token m is the bitmask of the tokens scanned up to and including m."""
    H, W = 2, 3
    expected_orders = {
        0: [0, 1, 2, 3, 4, 5],  # rows top->bottom, x ascending
        1: [2, 1, 0, 5, 4, 3],  # rows top->bottom, x descending
        2: [0, 3, 1, 4, 2, 5],  # columns left->right, y ascending
        3: [3, 0, 4, 1, 5, 2],  # columns left->right, y descending
    }
    L = H * W
    q = np.ones((1, L, 1, 1))
    k = np.ones((1, L, 1, 1))
    v = (2.0 ** np.arange(L)).reshape(1, L, 1, 1)
    lg = np.zeros((1, L, 1, 1))
    for d, order in expected_orders.items():
        assert [oracle.scan_token(s, d, H, W) for s in range(L)] == order
        assert list(oracle.scan_order(d, H, W)) == order
        out = oracle.gla_fwd(q, k, v, lg, H, W, d)[0, :, 0, 0]
        mask = 0
        for m in order:
            mask |= 1 << m
            assert out[m] == mask


def test_direction_identities():
    """R->L(G) = flipW(L->R(flipW G)); T->B(G) = L->R on the transposed grid; B->T(G) = flipH(T->B(flipH G))."""
    H, W = 5, 7
    q, k, v, lg = rand_case(2, H * W, 2, 4, 3, seed=6)

    def grid(x):
        return x.reshape(x.shape[0], H, W, *x.shape[2:])

    def flat(x):
        return x.reshape(x.shape[0], -1, *x.shape[3:])

    def flip_w(x):
        return flat(grid(x)[:, :, ::-1])

    def flip_h(x):
        return flat(grid(x)[:, ::-1])

    def transpose(x):
        return flat(np.swapaxes(grid(x), 1, 2))

    def untranspose(x):  # (W, H) grid back to (H, W)
        return flat(np.swapaxes(x.reshape(x.shape[0], W, H, *x.shape[2:]), 1, 2))

    r2l = oracle.gla_fwd(q, k, v, lg, H, W, 1)
    via = flip_w(oracle.gla_fwd(flip_w(q), flip_w(k), flip_w(v), flip_w(lg), H, W, 0))
    np.testing.assert_array_equal(r2l, via)

    t2b = oracle.gla_fwd(q, k, v, lg, H, W, 2)
    via = untranspose(oracle.gla_fwd(transpose(q), transpose(k), transpose(v), transpose(lg), W, H, 0))
    np.testing.assert_array_equal(t2b, via)

    b2t = oracle.gla_fwd(q, k, v, lg, H, W, 3)
    via = flip_h(oracle.gla_fwd(flip_h(q), flip_h(k), flip_h(v), flip_h(lg), H, W, 2))
    np.testing.assert_array_equal(b2t, via)


# ---------------------------------------------------------------- invariants
def test_causality():
    """Changing tokens after scan position s leaves every output at positions <= s unchanged."""
    H, W = 6, 6
    q, k, v, lg = rand_case(1, H * W, 2, 4, 4, seed=7)
    for d in range(4):
        order = oracle.scan_order(d, H, W)
        base = oracle.gla_fwd(q, k, v, lg, H, W, d)
        s = 17
        later = order[s + 1:]
        q2, k2, v2, lg2 = (x.copy() for x in (q, k, v, lg))
        rng = np.random.default_rng(99)
        for x in (q2, k2, v2):
            x[:, later] = rng.standard_normal(x[:, later].shape)
        lg2[:, later] = -rng.random(lg2[:, later].shape)
        pert = oracle.gla_fwd(q2, k2, v2, lg2, H, W, d)
        np.testing.assert_array_equal(base[:, order[: s + 1]], pert[:, order[: s + 1]])
        assert not np.allclose(base[:, later], pert[:, later])


def test_linear_in_v_and_columns_independent():
    H, W = 4, 8
    q, k, v, lg = rand_case(1, H * W, 2, 5, 6, seed=8)
    _, _, v2, _ = rand_case(1, H * W, 2, 5, 6, seed=9)
    a = oracle.gla_fwd(q, k, v, lg, H, W, 1)
    b = oracle.gla_fwd(q, k, v2, lg, H, W, 1)
    c = oracle.gla_fwd(q, k, 2.0 * v - 3.0 * v2, lg, H, W, 1)
    np.testing.assert_allclose(c, 2.0 * a - 3.0 * b, rtol=1e-11, atol=1e-11)
    # column j of the output depends on column j of v only (decay is key-side only)
    v3 = v.copy()
    v3[..., 2] += 1.0
    d = oracle.gla_fwd(q, k, v3, lg, H, W, 1)
    np.testing.assert_array_equal(np.delete(d, 2, axis=-1), np.delete(a, 2, axis=-1))
    assert not np.allclose(d[..., 2], a[..., 2])


def test_thread_count_does_not_change_result():
    w = WORKLOADS["tiny"]
    q, k, v, lg = make_inputs(w, 123)
    a = oracle.gla_fwd(q, k, v, lg, w.H, w.W, 0, threads=1)
    b = oracle.gla_fwd(q, k, v, lg, w.H, w.W, 0, threads=4)
    np.testing.assert_array_equal(a, b)


def test_rejects_bad_arguments():
    q, k, v, lg = rand_case(1, 6, 1, 2, 2, seed=1)
    with pytest.raises(ValueError):
        oracle.gla_fwd(q, k, v, lg, 2, 3, direction=4)
    with pytest.raises(ValueError):
        oracle.gla_fwd(q, k, v, lg, 2, 4, direction=0)


# ---------------------------------------------------------------- stored fixtures
def test_golden_fixtures():
    """Sampled outputs stored by tests/golden/make_golden.py (which calls only the oracle)."""
    path = os.path.join(GOLDEN, "oracle_samples.json")
    with open(path) as f:
        fixtures = json.load(f)
    assert fixtures
    for fx in fixtures:
        w = WORKLOADS[fx["workload"]].with_(**fx.get("override", {}))
        q, k, v, lg = make_inputs(w, fx["seed"])
        out = oracle.gla_fwd(q, k, v, lg, w.H, w.W, fx["direction"])
        idx = tuple(np.array(fx["index"]).T)
        np.testing.assert_allclose(out[idx], np.array(fx["value"]), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(np.sqrt(np.mean(out ** 2)), fx["rms"], rtol=1e-12)


# ---------------------------------------------------------------- the pins bite
def _mutant(q, k, v, lg, H, W, direction, mutation):
    """Sequential recurrence with one planted mistake (numpy, float64)."""
    order = oracle.scan_order(direction, H, W)
    if mutation == "wrong_order":
        order = order[::-1]
    B, L, heads, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((B, L, heads, dv))
    for b in range(B):
        for h in range(heads):
            S = np.zeros((dk, dv))
            prev = None
            for s in range(L):
                m = order[s]
                g = np.exp(lg[b, m, h])
                if mutation == "decay_after_add":
                    S = g[:, None] * (S + np.outer(k[b, m, h], v[b, m, h]))
                elif mutation == "value_side_decay":
                    gv = np.exp(lg[b, m, h][: dv]) if dv <= dk else np.ones(dv)
                    S = S * gv[None, :] + np.outer(k[b, m, h], v[b, m, h])
                elif mutation == "sign":
                    S = np.exp(-lg[b, m, h])[:, None] * S + np.outer(k[b, m, h], v[b, m, h])
                elif mutation == "output_before_update":
                    if prev is None:
                        prev = np.zeros((dk, dv))
                    out[b, m, h] = q[b, m, h] @ S / np.sqrt(dk)
                    S = g[:, None] * S + np.outer(k[b, m, h], v[b, m, h])
                    continue
                else:
                    S = g[:, None] * S + np.outer(k[b, m, h], v[b, m, h])
                scale = np.sqrt(dv) if mutation == "scale_dv" else np.sqrt(dk)
                out[b, m, h] = q[b, m, h] @ S / scale
    return out


@pytest.mark.parametrize("mutation", ["none", "decay_after_add", "value_side_decay", "sign",
                                      "output_before_update", "scale_dv", "wrong_order"])
def test_pins_reject_planted_mistakes(mutation):
    """The brute-force pin accepts the correct recurrence and rejects each planted mistake."""
    H, W = 2, 4
    q, k, v, lg = rand_case(1, H * W, 1, 4, 3, seed=11)
    ref = oracle.gla_fwd_bruteforce(q, k, v, lg, H, W, 1)
    got = _mutant(q, k, v, lg, H, W, 1, mutation)
    if mutation == "none":
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    else:
        assert not np.allclose(got, ref, rtol=1e-6, atol=1e-6)
