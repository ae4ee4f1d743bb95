"""Pins for the oracle's permutation (CPU only).

Passages: dots.llm1 Technical Report, §3.2 "Efficient implementation of
Grouped GEMM" (each expert's token segment M_i is aligned to a fixed block)
and §Architecture "Load balancing" (no token is dropped).  Checked against a
brute-force bucket sort written with Python's stable ``sorted`` and against
the invariants the passages fix.
"""
import numpy as np
import pytest

import oracle


def _random_idx(rng, T, E, k):
    return np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)


def _bruteforce(idx, E, P, cap):
    T, k = idx.shape
    pairs = sorted(((int(idx[t, j]), t, j) for t in range(T) for j in range(k)))
    counts = [sum(1 for p in pairs if p[0] == e) for e in range(E)]
    offsets = [0]
    for e in range(E):
        offsets.append(offsets[-1] + -(-counts[e] // P) * P)
    sorted_ids = [-1] * cap
    row_of = np.full((T, k), -1, np.int32)
    fill = [0] * E
    for e, t, j in pairs:
        pos = offsets[e] + fill[e]
        fill[e] += 1
        sorted_ids[pos] = t
        row_of[t, j] = pos
    return counts, offsets, sorted_ids, row_of


@pytest.mark.parametrize("T,E,k,P", [(1, 4, 1, 16), (7, 4, 2, 1), (64, 8, 2, 16), (50, 16, 6, 8),
                                     (33, 5, 5, 128), (100, 12, 3, 64)])
def test_permute_matches_bruteforce(T, E, k, P):
    rng = np.random.default_rng(T * 31 + E)
    idx = _random_idx(rng, T, E, k)
    cap = T * k + E * (P - 1)
    got = oracle.permute(idx, E, P, cap)
    counts, offsets, sorted_ids, row_of = _bruteforce(idx, E, P, cap)
    assert list(got["counts"]) == counts
    assert list(got["offsets"]) == offsets
    assert list(got["sorted_ids"]) == sorted_ids
    assert np.array_equal(got["row_of"], row_of)
    assert got["total"] == offsets[-1]


def test_permute_invariants():
    rng = np.random.default_rng(9)
    T, E, k, P = 300, 16, 4, 32
    idx = _random_idx(rng, T, E, k)
    # make expert 3 empty
    for t in range(T):
        if 3 in idx[t]:
            free = [e for e in range(E) if e not in idx[t] and e != 3]
            idx[t][list(idx[t]).index(3)] = free[0]
    cap = T * k + E * (P - 1)
    r = oracle.permute(idx, E, P, cap)
    c, off = r["counts"], r["offsets"]
    assert c.sum() == T * k                                  # no token dropped
    assert c[3] == 0 and off[4] == off[3]                     # empty expert: zero rows
    assert np.all((off[1:] - off[:-1]) == -(-c // P) * P)     # segments padded to P
    assert np.all(off % P == 0) and r["total"] == off[-1]
    so, ro = r["sorted_ids"], r["row_of"]
    # every (t, j) once, and it points back to its token
    assert len(set(ro.ravel().tolist())) == T * k
    assert np.all(so[ro] == np.arange(T)[:, None])
    # each row sits inside its expert's segment; tokens ascend inside a segment
    for e in range(E):
        seg = so[off[e]:off[e + 1]]
        real = seg[:c[e]]
        assert np.all(np.diff(real) > 0)
        assert np.all(seg[c[e]:] == -1)
        assert all(e in idx[t] for t in real)
    assert np.all(so[r["total"]:] == -1)


def test_permute_without_padding_is_plain_counting_sort():
    rng = np.random.default_rng(11)
    idx = _random_idx(rng, 40, 6, 3)
    r = oracle.permute(idx, 6, 1, 120)
    assert np.array_equal(r["offsets"], np.concatenate([[0], np.cumsum(np.bincount(idx.ravel(), minlength=6))]))
    flat_e = idx.ravel()
    flat_t = np.repeat(np.arange(40), 3)
    order = np.lexsort((flat_t, flat_e))
    assert np.array_equal(r["sorted_ids"], flat_t[order])


def test_permute_rejects_overflowing_capacity():
    idx = np.array([[0], [0], [1]], np.int32)
    with pytest.raises(ValueError):
        oracle.permute(idx, 2, 16, 20)  # needs 32 rows
