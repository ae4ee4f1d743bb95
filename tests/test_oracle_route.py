"""Pins for the oracle's gate and router (CPU only).

Passages: dots.llm1 Technical Report, §Architecture "Mixture of Experts layer"
(FP32 gating layer, top-6 of 128 routed experts) and "Load balancing" (bias
added to the affinity scores only to choose the top-k).  Each test checks the
oracle against something other than itself: numpy's matmul, closed forms of the
softmax, brute force over all k-subsets, hand-derived fixtures.
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_case(rng, T, d, E):
    x = synth.normal_bf16(7, 1, (T, d), 1.0)
    wg = synth.normal_f32(7, 2, (E, d), 0.05)
    return x, wg


def test_gate_logits_match_numpy_matmul():
    x, wg = _rand_case(None, 37, 96, 8)
    ref = synth.bf16_to_f32(x).astype(np.float64) @ wg.astype(np.float64).T
    got = oracle.gate_logits(x, wg)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_gate_logits_unit_rows_pick_columns():
    # x = identity rows (bf16 1.0 = 0x3F80): logit[t, e] = Wg[e, t] exactly.
    d, E = 16, 8
    x = np.zeros((d, d), dtype=np.uint16)
    x[np.arange(d), np.arange(d)] = 0x3F80
    wg = synth.normal_f32(3, 2, (E, d), 1.0)
    got = oracle.gate_logits(x, wg)
    assert np.array_equal(got, wg.T.astype(np.float64))


def test_softmax_two_experts_is_sigmoid():
    logits = np.array([[0.3, -1.1], [5.0, 5.0], [-2.0, 7.5]])
    p, idx, w, m = oracle.route(logits, np.zeros(2, np.float32), 1)
    for t in range(3):
        p0 = 1.0 / (1.0 + math.exp(logits[t, 1] - logits[t, 0]))
        assert abs(p[t, 0] - p0) < 1e-15 and abs(p[t, 1] - (1 - p0)) < 1e-15


def test_softmax_shift_invariance_and_ratios():
    rng = np.random.default_rng(0)
    logits = rng.normal(size=(20, 16)) * 3
    p, *_ = oracle.route(logits, np.zeros(16, np.float32), 4)
    p2, *_ = oracle.route(logits + 123.25, np.zeros(16, np.float32), 4)
    np.testing.assert_allclose(p, p2, rtol=1e-12)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    # closed form of the ratio: p_a / p_b = exp(l_a - l_b)
    np.testing.assert_allclose(p[:, 3] / p[:, 7], np.exp(logits[:, 3] - logits[:, 7]), rtol=1e-12)


def _bruteforce_topk(s, k):
    """The chosen set maximises the sum of biased scores; among equal sums the
    set with the lowest indices wins.  Order: s descending, ties by index."""
    E = len(s)
    best = None
    for sub in itertools.combinations(range(E), k):
        key = (-sum(s[e] for e in sub), sub)
        if best is None or key < best:
            best = key
    chosen = best[1]
    return sorted(chosen, key=lambda e: (-s[e], e))


@pytest.mark.parametrize("k", [1, 2, 3, 5])
def test_topk_matches_bruteforce_over_subsets(k):
    rng = np.random.default_rng(k)
    E, T = 8, 60
    logits = rng.normal(size=(T, E)) * 2
    # quantised bias + some all-equal logits rows create exact ties
    bias = (rng.integers(-2, 3, size=E) * 0.125).astype(np.float32)
    logits[::5] = 0.0
    p, idx, w, margin = oracle.route(logits, bias, k)
    for t in range(T):
        s = [p[t, e] + float(bias[e]) for e in range(E)]
        assert list(idx[t]) == _bruteforce_topk(s, k), t
        chosen = set(idx[t])
        rest = [s[e] for e in range(E) if e not in chosen]
        assert margin[t] == pytest.approx(s[idx[t, -1]] - max(rest), abs=1e-15)


def test_weights_are_unbiased_probs_renormalised():
    rng = np.random.default_rng(2)
    E, k, T = 16, 6, 40
    logits = rng.normal(size=(T, E))
    bias = rng.uniform(-0.05, 0.05, size=E).astype(np.float32)
    p, idx, w, _ = oracle.route(logits, bias, k)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-14)
    for t in range(T):
        sel = p[t, idx[t]]
        np.testing.assert_allclose(w[t], sel / sel.sum(), rtol=1e-14)
        assert len(set(idx[t])) == k and idx[t].min() >= 0 and idx[t].max() < E


def test_bias_changes_selection_not_weights():
    rng = np.random.default_rng(3)
    E, k, T = 12, 3, 30
    logits = rng.normal(size=(T, E))
    b = rng.uniform(-0.02, 0.02, size=E).astype(np.float32)
    # a constant shift of every bias keeps the selection and the weights
    _, i1, w1, _ = oracle.route(logits, b, k)
    _, i2, w2, _ = oracle.route(logits, b + np.float32(0.25), k)
    assert np.array_equal(i1, i2)
    np.testing.assert_allclose(w1, w2, rtol=1e-14)
    # forcing a set with a huge bias: weights are still the unbiased p renormalised
    force = np.zeros(E, np.float32)
    force[[1, 4, 9]] = 10.0
    p, i3, w3, _ = oracle.route(logits, force, k)
    for t in range(T):
        assert set(i3[t]) == {1, 4, 9}
        np.testing.assert_allclose(w3[t], p[t, i3[t]] / p[t, [1, 4, 9]].sum(), rtol=1e-14)


def test_special_cases_k_equals_E_and_k1():
    rng = np.random.default_rng(4)
    E, T = 8, 25
    logits = rng.normal(size=(T, E))
    p, idx, w, margin = oracle.route(logits, np.zeros(E, np.float32), E)
    for t in range(T):
        assert sorted(idx[t]) == list(range(E))
        np.testing.assert_allclose(w[t], p[t, idx[t]], rtol=1e-14)
    assert np.all(np.isinf(margin))
    _, idx1, w1, _ = oracle.route(logits, np.zeros(E, np.float32), 1)
    assert np.array_equal(idx1[:, 0], np.argmax(logits, axis=1))
    assert np.all(w1 == 1.0)


def _golden_cases():
    cases = []
    with open(os.path.join(GOLDEN, "route_hand.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, k, lg, b, i, w, m = [c.strip() for c in line.split("|")]
            cases.append((name, int(k), [float(v) for v in lg.split()],
                          [float(v) for v in b.split()], [int(v) for v in i.split()],
                          [float(v) for v in w.split()], float(m)))
    return cases


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c[0])
def test_hand_derived_routing_fixture(case):
    name, k, lg, b, i, w, m = case
    _, idx, wt, margin = oracle.route(np.array([lg]), np.array(b, np.float32), k)
    assert list(idx[0]) == i
    np.testing.assert_allclose(wt[0], w, rtol=1e-12)
    if math.isinf(m):
        assert math.isinf(margin[0])
    else:
        assert abs(margin[0] - m) < 1e-7  # bias is stored in f32


def _fp32_bits_case(T=4, d=4096, E=8):
    """x = +1, -1, +1, ... (bf16) and Wg = 1 + e * 2^-22 on the even columns, 1 on the odd
    ones: the weights differ only below bf16's 8-bit significand."""
    sign = np.where(np.arange(d) % 2 == 0, 1.0, -1.0).astype(np.float32)
    x = np.tile((sign.view(np.uint32) >> 16).astype(np.uint16), (T, 1))
    wg = np.ones((E, d), np.float32)
    wg[:, 0::2] += (np.arange(E, dtype=np.float32) * np.float32(2.0 ** -22))[:, None]
    return x, wg


def test_gate_logits_keep_fp32_weight_bits():
    # closed form: logit_e = (d / 2) * e * 2^-22 = e * 2^-11 exactly (FP32 gate of the pages,
    # §Architecture "Mixture of Experts layer"); a bf16 copy of Wg would make all logits 0
    x, wg = _fp32_bits_case()
    logits = oracle.gate_logits(x, wg)
    assert np.array_equal(logits, np.tile(np.arange(8) * 2.0 ** -11, (4, 1)))
    wg_bf16 = (wg.view(np.uint32) + 0x8000 & 0xFFFF0000).view(np.float32)
    assert np.all(oracle.gate_logits(x, wg_bf16) == 0.0)
    _, idx, _, margin = oracle.route(logits, np.zeros(8, np.float32), 3)
    assert idx.tolist() == [[7, 6, 5]] * 4
    assert np.all(margin > 5e-5)
