"""Pins of the oracle's router backward and bias update (CPU only).

Passages: dots.llm1 Technical Report, §Architecture "Mixture of Experts layer"
(FP32 gate; the combine weights are the affinities of the chosen experts) and
"Load balancing" (a per-expert bias, used only to choose the top-k, adjusted
during training to keep the loads balanced).  The backward is the derivative
of the forward the oracle states; it is pinned here by finite differences
through the oracle's own forward (gate_logits + route, which have their own
pins), by the softmax Jacobian in matrix form for k = E, and by invariants.
"""
import numpy as np
import pytest

import oracle
import synth


def _case(T=5, d=64, E=8, k=3, seed=11):
    x = synth.normal_bf16(seed, 1, (T, d), 0.5)
    wg = synth.normal_f32(seed, 2, (E, d), 0.3)
    dw = synth.normal_f32(seed, 6, (T, k), 1.0).astype(np.float64)
    bias = np.zeros(E, np.float32)
    return x, wg, dw, bias


def _loss(x, wg, bias, k, dw, idx_ref):
    """L = sum_{t,j} dw[t,j] * w[t,j] through the forward oracle; the selection
    must stay the one being differentiated."""
    _, idx, w, _ = oracle.route(oracle.gate_logits(x, wg), bias, k)
    assert np.array_equal(idx, idx_ref), "a perturbation changed the selection"
    return float(np.sum(dw * w))


def test_dlogits_match_finite_differences_of_route():
    x, wg, dw, bias = _case()
    k = dw.shape[1]
    logits = oracle.gate_logits(x, wg)
    _, idx, _, margin = oracle.route(logits, bias, k)
    assert margin.min() > 1e-3
    dl, _, _ = oracle.router_bwd(x, wg, idx, dw)
    h = 1e-6
    fd = np.zeros_like(logits)
    for t in range(logits.shape[0]):
        for e in range(logits.shape[1]):
            lp, lm = logits.copy(), logits.copy()
            lp[t, e] += h
            lm[t, e] -= h
            _, ip, wp, _ = oracle.route(lp, bias, k)
            _, im, wm, _ = oracle.route(lm, bias, k)
            assert np.array_equal(ip, idx) and np.array_equal(im, idx)
            fd[t, e] = (np.sum(dw * wp) - np.sum(dw * wm)) / (2 * h)
    np.testing.assert_allclose(dl, fd, rtol=1e-6, atol=1e-9)


def test_dwg_matches_finite_differences():
    x, wg, dw, bias = _case()
    k = dw.shape[1]
    _, idx, _, _ = oracle.route(oracle.gate_logits(x, wg), bias, k)
    _, _, dwg = oracle.router_bwd(x, wg, idx, dw)
    rng = np.random.default_rng(3)
    h = np.float32(2.0 ** -14)  # wg +- h is exact in f32 for these magnitudes
    for _ in range(24):
        e, c = int(rng.integers(wg.shape[0])), int(rng.integers(wg.shape[1]))
        wp, wm = wg.copy(), wg.copy()
        wp[e, c] += h
        wm[e, c] -= h
        assert float(wp[e, c]) - float(wg[e, c]) == float(h)
        fd = (_loss(x, wp, bias, k, dw, idx) - _loss(x, wm, bias, k, dw, idx)) / (2 * float(h))
        assert fd == pytest.approx(dwg[e, c], rel=1e-5, abs=1e-9)


def test_dx_matches_finite_differences():
    x, wg, dw, bias = _case()
    k = dw.shape[1]
    _, idx, _, _ = oracle.route(oracle.gate_logits(x, wg), bias, k)
    _, dx, _ = oracle.router_bwd(x, wg, idx, dw)
    xf = synth.bf16_to_f32(x)
    rng = np.random.default_rng(4)
    h = 2.0 ** -8  # x +- h stays a bf16 value while |x| < 0.99
    checked = 0
    while checked < 24:
        t, c = int(rng.integers(x.shape[0])), int(rng.integers(x.shape[1]))
        if abs(xf[t, c]) >= 0.99:
            continue
        to_bits = lambda v: (np.array([v], np.float32).view(np.uint32) >> 16).astype(np.uint16)[0]
        xp, xm = x.copy(), x.copy()
        xp[t, c] = to_bits(xf[t, c] + h)
        xm[t, c] = to_bits(xf[t, c] - h)
        assert synth.bf16_to_f32(xp)[t, c] - xf[t, c] == h
        assert xf[t, c] - synth.bf16_to_f32(xm)[t, c] == h
        fd = (_loss(xp, wg, bias, k, dw, idx) - _loss(xm, wg, bias, k, dw, idx)) / (2 * h)
        assert fd == pytest.approx(dx[t, c], rel=1e-4, abs=1e-8)
        checked += 1


def test_k_equals_E_is_the_softmax_jacobian():
    # all experts chosen: w = p (the renormaliser is 1), so dlogit = (diag(p) - p p^T) dL/dp
    x, wg, _, bias = _case(E=6, k=6)
    dw = synth.normal_f32(5, 6, (x.shape[0], 6), 1.0).astype(np.float64)
    p, idx, _, _ = oracle.route(oracle.gate_logits(x, wg), bias, 6)
    dl, _, _ = oracle.router_bwd(x, wg, idx, dw)
    for t in range(x.shape[0]):
        dp = np.zeros(6)
        dp[idx[t]] = dw[t]
        J = np.diag(p[t]) - np.outer(p[t], p[t])
        np.testing.assert_allclose(dl[t], J @ dp, rtol=1e-12, atol=1e-15)


def test_k1_has_no_gradient_and_rows_sum_to_zero():
    x, wg, _, bias = _case(k=1)
    dw = np.ones((x.shape[0], 1))
    _, idx, _, _ = oracle.route(oracle.gate_logits(x, wg), bias, 1)
    dl, dx, dwg = oracle.router_bwd(x, wg, idx, dw)
    assert np.all(dl == 0.0) and np.all(dx == 0.0) and np.all(dwg == 0.0)  # w == 1 always
    x, wg, dw, bias = _case(T=9, E=16, k=4, seed=12)
    _, idx, _, _ = oracle.route(oracle.gate_logits(x, wg), bias, 4)
    dl, _, _ = oracle.router_bwd(x, wg, idx, dw)
    np.testing.assert_allclose(dl.sum(axis=1), 0.0, atol=1e-15)  # softmax shift invariance


def test_bias_update_hand_case():
    # T = 4 tokens, k = 2, E = 4: mean load 2.  loads: e0 = 4, e1 = 2, e2 = 2, e3 = 0
    idx = np.array([[0, 1], [0, 2], [0, 1], [0, 2]], np.int32)
    bias = np.array([0.5, -0.25, 0.0, 1.0], np.float32)
    out = oracle.bias_update(idx, 4, bias, 0.125)
    assert out.tolist() == [0.375, -0.25, 0.0, 1.125]
    # the sum of two f32 values is exact in double: rounding it once gives the f32 result
    out = oracle.bias_update(idx, 4, np.full(4, 0.1, np.float32), 1e-3)
    assert out[0] == float(np.float32(0.1)) - float(np.float32(1e-3))
