"""Pins of the oracle's sequence-wise balance loss (``oracle.seq_balance``).

Passage: dots.llm1 Technical Report, §Architecture "Load balancing": besides the
aux-loss-free bias, a sequence-wise balance loss keeps any single sequence from
extreme imbalance.  The pages give no formula; the reading is the one of the
report they cite for their method (DeepSeek-V3): per sequence, alpha times the
sum over experts of (load fraction x E / k) times (mean normalised affinity),
averaged over the batch's sequences.

The pins below do not restate that formula; they check results it fixes:
  * k = E (every expert picked by every token): the loss is exactly alpha for
    any logits (a wrong load or affinity normalisation breaks this);
  * uniform affinities with perfectly balanced picks: alpha;
  * every token on the same k experts with all affinity on them: alpha E / k;
  * per-sequence segmentation, a short last sequence, and the mean over
    sequences, from sequences built to have those known values;
  * the gradient against central finite differences of the loss (picks held
    fixed), and its rows summing to zero (softmax gradient);
  * tokens may be reordered inside a sequence, not across sequences.
"""
import numpy as np
import pytest

import oracle

ALPHA = 1e-2
NEG = -1e4  # exp(NEG - max) is 0 in double: that expert's affinity is exactly 0


def _balanced_idx(L, E, k):
    # token t picks (t k + j) mod E: every expert k L / E times when E | k L
    return np.array([[(t * k + j) % E for j in range(k)] for t in range(L)], np.int32)


def test_every_expert_picked_gives_alpha():
    rng = np.random.default_rng(1)
    for T, E, L in [(37, 8, 37), (64, 16, 64), (10, 4, 10)]:
        lg = rng.normal(0, 3, (T, E))
        idx = np.tile(np.arange(E, dtype=np.int32), (T, 1))
        loss, _ = oracle.seq_balance(lg, idx, L, ALPHA)
        assert loss == pytest.approx(ALPHA, rel=1e-13)


def test_uniform_affinity_balanced_picks_gives_alpha():
    E, k, L = 8, 2, 16
    idx = _balanced_idx(L, E, k)
    loss, _ = oracle.seq_balance(np.zeros((L, E)), idx, L, ALPHA)
    assert loss == pytest.approx(ALPHA, rel=1e-13)


def test_collapsed_routing_gives_alpha_e_over_k():
    E, k, L = 8, 2, 16
    lg = np.full((L, E), NEG)
    lg[:, :k] = 0.0  # affinity 1/k on experts 0..k-1, 0 elsewhere
    idx = np.tile(np.arange(k, dtype=np.int32), (L, 1))
    loss, _ = oracle.seq_balance(lg, idx, L, ALPHA)
    assert loss == pytest.approx(ALPHA * E / k, rel=1e-13)


def test_sequences_are_scored_separately_and_averaged():
    E, k, L = 8, 2, 16
    bal_lg, bal_idx = np.zeros((L, E)), _balanced_idx(L, E, k)
    col_lg = np.full((L, E), NEG)
    col_lg[:, :k] = 0.0
    col_idx = np.tile(np.arange(k, dtype=np.int32), (L, 1))
    # [balanced | collapsed | 5-token collapsed tail]
    lg = np.concatenate([bal_lg, col_lg, col_lg[:5]])
    idx = np.concatenate([bal_idx, col_idx, col_idx[:5]])
    loss, _ = oracle.seq_balance(lg, idx, L, ALPHA)
    assert loss == pytest.approx((ALPHA + 2 * ALPHA * E / k) / 3, rel=1e-13)
    # the same tokens as one sequence are one mixed sequence, not the mean of three
    one, _ = oracle.seq_balance(lg, idx, len(lg), ALPHA)
    assert one != pytest.approx(loss, rel=1e-6)


def test_gradient_matches_finite_differences():
    rng = np.random.default_rng(2)
    T, E, k, L = 23, 8, 3, 10  # three sequences, the last of 3 tokens
    lg = rng.normal(0, 1.5, (T, E))
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    _, dl = oracle.seq_balance(lg, idx, L, ALPHA)
    h = 1e-5
    for t, e in [(0, 0), (4, 7), (9, 3), (10, 1), (15, 5), (21, 2), (22, 6)]:
        lp, lm = lg.copy(), lg.copy()
        lp[t, e] += h
        lm[t, e] -= h
        fd = (oracle.seq_balance(lp, idx, L, ALPHA, want_grad=False)[0] -
              oracle.seq_balance(lm, idx, L, ALPHA, want_grad=False)[0]) / (2 * h)
        assert dl[t, e] == pytest.approx(fd, rel=1e-6, abs=1e-12)
    np.testing.assert_allclose(dl.sum(axis=1), 0.0, atol=1e-17)


def test_order_inside_a_sequence_does_not_matter_across_does():
    rng = np.random.default_rng(3)
    T, E, k, L = 32, 8, 2, 16
    lg = rng.normal(0, 1, (T, E))
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    base, _ = oracle.seq_balance(lg, idx, L, ALPHA)
    inside = np.concatenate([rng.permutation(L), L + rng.permutation(L)])
    assert oracle.seq_balance(lg[inside], idx[inside], L, ALPHA)[0] == pytest.approx(base,
                                                                                 rel=1e-13)
    across = rng.permutation(T)
    assert oracle.seq_balance(lg[across], idx[across], L, ALPHA)[0] != pytest.approx(base,
                                                                                 rel=1e-9)


def test_router_bwd_adds_the_extra_term_before_dx_and_dwg():
    # dl_extra enters dX = dl Wg and dWg = dl^T X linearly: the extra term alone
    # (dw = 0) gives dX = dl_extra Wg exactly as a plain matrix product of it
    rng = np.random.default_rng(4)
    T, d, E, k = 12, 16, 8, 2
    x = (rng.normal(0, 1, (T, d)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    wg = rng.normal(0, 0.1, (E, d)).astype(np.float32)
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    extra = rng.normal(0, 1e-3, (T, E))
    dl, dx, dwg = oracle.router_bwd(x, wg, idx, np.zeros((T, k)), dl_extra=extra)
    np.testing.assert_array_equal(dl, extra)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    np.testing.assert_allclose(dx, extra @ wg.astype(np.float64), rtol=1e-12, atol=1e-18)
    np.testing.assert_allclose(dwg, extra.T @ xf, rtol=1e-12, atol=1e-18)
