"""Pins for the oracle's backward (CPU only).

The layer of the dots.llm1 Technical Report (§Architecture "Mixture of Experts
layer") is trained, so its gradients are part of the path.  The oracle's
analytic gradients are pinned by FP64 central finite differences of the
oracle's own forward (the double-precision form, no bf16 storage rounding) on
the scalar L = <dOut, out>.  The forward is pinned separately, so a wrong sign,
index or dropped term in the backward fails here.
"""
import numpy as np
import pytest

import oracle

T, D, E, K, S, I = 5, 8, 4, 2, 1, 4
H_FD = 1e-6


@pytest.fixture(scope="module")
def case():
    rng = np.random.default_rng(21)
    x = rng.normal(size=(T, D))
    w1 = rng.normal(size=(E + S, 2 * I, D)) * 0.4
    w2 = rng.normal(size=(E + S, D, I)) * 0.4
    dout = rng.normal(size=(T, D))
    idx = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    w = rng.uniform(0.2, 1.0, size=(T, K))
    return x, w1, w2, dout, idx, w


def _loss(x, w1, w2, dout, idx, w):
    out = oracle.layer_fwd(x, idx, w, w1, w2, S=S, rnd=False)
    return float(np.sum(out * dout))


def _fd(f, arr, positions):
    g = []
    for pos in positions:
        old = arr[pos]
        arr[pos] = old + H_FD
        lp = f()
        arr[pos] = old - H_FD
        lm = f()
        arr[pos] = old
        g.append((lp - lm) / (2 * H_FD))
    return np.array(g)


def _check(an, fd):
    err = np.max(np.abs(an - fd)) / max(np.max(np.abs(fd)), 1e-30)
    assert err < 1e-6, (err, an, fd)


def test_dx_and_dw_match_finite_differences(case):
    x, w1, w2, dout, idx, w = case
    dx, dw = oracle.layer_bwd(x, idx, w, w1, w2, dout, S=S, rnd=False)
    f = lambda: _loss(x, w1, w2, dout, idx, w)
    pos = [(t, c) for t in range(T) for c in range(D)]
    _check(dx.ravel(), _fd(f, x, pos))
    posw = [(t, j) for t in range(T) for j in range(K)]
    _check(dw.ravel(), _fd(f, w, posw))


@pytest.mark.parametrize("grp", [0, 2, E])  # routed experts and the shared one
def test_dW_match_finite_differences(case, grp):
    x, w1, w2, dout, idx, w = case
    dw1, dw2 = oracle.group_dw(x, idx, w, w1, w2, dout, S=S, grp=grp, rnd=False)
    f = lambda: _loss(x, w1, w2, dout, idx, w)
    pos1 = [(grp, i, c) for i in range(2 * I) for c in range(D)]
    _check(dw1.ravel(), _fd(f, w1, pos1))
    pos2 = [(grp, r, c) for r in range(D) for c in range(I)]
    _check(dw2.ravel(), _fd(f, w2, pos2))


def test_unused_expert_has_zero_dW(case):
    x, w1, w2, dout, idx, w = case
    unused = [e for e in range(E) if e not in idx]
    if not unused:
        idx = idx.copy()
        idx[idx == 3] = [e for e in range(E) if e != 3][0]
        unused = [3]
    dw1, dw2 = oracle.group_dw(x, idx, w, w1, w2, dout, S=S, grp=unused[0], rnd=False)
    assert np.all(dw1 == 0) and np.all(dw2 == 0)


def test_selected_entries_equal_full_gradient(case):
    x, w1, w2, dout, idx, w = case
    full1, full2 = oracle.group_dw(x, idx, w, w1, w2, dout, S=S, grp=1, rnd=False)
    rows, cols = [7, 0, 5], [3, 1]
    sub1, sub2 = oracle.group_dw(x, idx, w, w1, w2, dout, S=S, grp=1, w1_rows=rows,
                                 w2_cols=cols, rnd=False)
    np.testing.assert_array_equal(sub1, full1[rows])
    np.testing.assert_array_equal(sub2, full2[:, cols])


def test_bf16_inputs_route_through_same_gradient():
    # The bf16 entry points widen exactly, so on bf16-representable inputs they
    # agree with the double entry points (rounding of H/Y switched off).
    import synth
    xb = synth.normal_bf16(5, 1, (T, D), 1.0)
    w1b = synth.normal_bf16(5, 4, (E + S, 2 * I, D), 0.4)
    w2b = synth.normal_bf16(5, 5, (E + S, D, I), 0.4)
    db = synth.normal_bf16(5, 6, (T, D), 1.0)
    f = lambda h: synth.bf16_to_f32(h).astype(np.float64)
    rng = np.random.default_rng(3)
    idx = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    w = rng.uniform(0.2, 1.0, size=(T, K))
    a = oracle.layer_bwd(xb, idx, w, w1b, w2b, db, S=S, rnd=False)
    b = oracle.layer_bwd(f(xb), idx, w, f(w1b), f(w2b), f(db), S=S, rnd=False)
    # equal up to the summation order the compiler picks for each instantiation
    np.testing.assert_allclose(a[0], b[0], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(a[1], b[1], rtol=1e-13, atol=1e-15)
