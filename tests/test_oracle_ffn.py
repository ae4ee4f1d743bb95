"""Pins for the oracle's expert FFN and layer forward (CPU only).

Passage: dots.llm1 Technical Report, §Architecture "Mixture of Experts layer":
every expert is a fine-grained two-layer FFN with SwiGLU; each token uses its
top-6 routed experts plus the 2 shared experts.  Checked against numpy's
matmul, a brute-force masked loop over all experts, a scalar closed form, the
dense-FFN special case, and a brute-force nearest-bf16 search.
"""
import math
import struct

import numpy as np
import pytest

import oracle
import synth


def _f(h):
    return synth.bf16_to_f32(h).astype(np.float64)


def _silu(v):
    return v / (1.0 + np.exp(-v))


def _numpy_expert(a, w1g, w2g):
    I = w2g.shape[1]
    A, W1, W2 = _f(a), _f(w1g), _f(w2g)
    g = A @ W1[:I].T
    u = A @ W1[I:].T
    h = _silu(g) * u
    return g, u, h, h @ W2.T


def _bf16_bits(v: float) -> int:
    return struct.unpack("<I", struct.pack("<f", v))[0] >> 16


def _nearest_bf16_bruteforce(v: float) -> float:
    """Nearest bf16 to v by trying the neighbours of a truncation; ties go to
    the candidate with an even last mantissa bit."""
    base = _bf16_bits(float(np.float32(v)))
    cands = []
    for b in (base - 2, base - 1, base, base + 1, base + 2):
        if 0 <= b < 0x10000:
            c = struct.unpack("<f", struct.pack("<I", b << 16))[0]
            if math.isfinite(c):
                cands.append((abs(c - v), b & 1, c))
    cands.sort()
    return cands[0][2]


def test_round_bf16_ties_and_bruteforce():
    assert oracle.round_bf16(1.0 + 2.0 ** -8) == 1.0                  # tie -> even (1.0)
    assert oracle.round_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6  # tie -> even
    assert oracle.round_bf16(-(1.0 + 3 * 2.0 ** -8)) == -(1.0 + 2.0 ** -6)
    assert oracle.round_bf16(1.0 + 2.0 ** -8 + 2.0 ** -30) == 1.0 + 2.0 ** -7
    rng = np.random.default_rng(5)
    for v in np.concatenate([rng.normal(size=300) * 10.0 ** rng.integers(-6, 6, size=300),
                             rng.uniform(-1, 1, size=100)]):
        assert oracle.round_bf16(float(v)) == _nearest_bf16_bruteforce(float(v)), v


def test_expert_fwd_matches_numpy():
    d, I, M = 64, 32, 9
    a = synth.normal_bf16(1, 1, (M, d), 1.0)
    w1 = synth.normal_bf16(1, 4, (2 * I, d), 0.1)
    w2 = synth.normal_bf16(1, 5, (d, I), 0.1)
    g, u, h, y = oracle.expert_fwd(a, w1, w2, rnd=False)
    rg, ru, rh, ry = _numpy_expert(a, w1, w2)
    for got, ref in ((g, rg), (u, ru), (h, rh), (y, ry)):
        np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-13)
    # storage rounding: H and Y are the nearest bf16 of the exact values
    _, _, hr, yr = oracle.expert_fwd(a, w1, w2, rnd=True)
    for v, vr in zip(h.ravel()[:200], hr.ravel()[:200]):
        assert vr == _nearest_bf16_bruteforce(v)
    assert np.max(np.abs(hr - h)) <= 2.0 ** -8 * np.max(np.abs(h))


def test_scalar_swiglu_closed_form():
    # d = 1, I = 1: y = w2 * silu(wg x) * (wu x), all inputs exact in bf16
    bits = lambda v: np.array([[_bf16_bits(v)]], np.uint16)
    x, wg, wu, w2 = 2.0, 0.5, 3.0, 0.25
    w1 = np.array([[_bf16_bits(wg)], [_bf16_bits(wu)]], np.uint16)
    g, u, h, y = oracle.expert_fwd(bits(x), w1, bits(w2), rnd=False)
    G, U = wg * x, wu * x
    H = G / (1 + math.exp(-G)) * U
    assert g[0, 0] == G and u[0, 0] == U
    assert abs(h[0, 0] - H) < 1e-15 and abs(y[0, 0] - w2 * H) < 1e-15


def test_dense_ffn_special_case():
    # E = 1 routed expert, k = 1, no shared expert: the layer is one dense SwiGLU FFN.
    T, d, I = 12, 32, 16
    x = synth.normal_bf16(2, 1, (T, d), 1.0)
    w1 = synth.normal_bf16(2, 4, (1, 2 * I, d), 0.1)
    w2 = synth.normal_bf16(2, 5, (1, d, I), 0.1)
    idx = np.zeros((T, 1), np.int32)
    w = np.ones((T, 1))
    out = oracle.layer_fwd(x, idx, w, w1, w2, S=0, rnd=False)
    *_, ref = _numpy_expert(x, w1[0], w2[0])
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-13)


def test_layer_matches_masked_loop_over_all_experts():
    T, d, E, k, S, I = 20, 32, 6, 2, 2, 16
    x = synth.normal_bf16(3, 1, (T, d), 1.0)
    w1 = synth.normal_bf16(3, 4, (E + S, 2 * I, d), 0.1)
    w2 = synth.normal_bf16(3, 5, (E + S, d, I), 0.1)
    rng = np.random.default_rng(1)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    w = rng.uniform(0.1, 1.0, size=(T, k))
    out, yr, ys = oracle.layer_fwd(x, idx, w, w1, w2, S=S, rnd=False, want_y=True)
    ref = np.zeros((T, d))
    for e in range(E + S):
        *_, ye = _numpy_expert(x, w1[e], w2[e])
        if e < E:
            mask = np.array([(w[t][list(idx[t]).index(e)] if e in idx[t] else 0.0) for t in range(T)])
        else:
            mask = np.ones(T)
        ref += mask[:, None] * ye
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)
    # token subsets give the same rows
    sub = oracle.layer_fwd(x, idx, w, w1, w2, S=S, tokens=[19, 3, 3], rnd=False)
    np.testing.assert_array_equal(sub, out[[19, 3, 3]])


def test_zero_gate_weights_give_zero_output():
    T, d, E, k, S, I = 8, 32, 4, 2, 1, 16
    x = synth.normal_bf16(4, 1, (T, d), 1.0)
    w1 = synth.normal_bf16(4, 4, (E + S, 2 * I, d), 0.1)
    w1[:, :I, :] = 0  # gate half zero -> silu(0) = 0 -> H = 0
    w2 = synth.normal_bf16(4, 5, (E + S, d, I), 0.1)
    idx = np.tile(np.array([[0, 3]], np.int32), (T, 1))
    out = oracle.layer_fwd(x, idx, np.full((T, k), 0.5), w1, w2, S=S)
    assert np.all(out == 0.0)
