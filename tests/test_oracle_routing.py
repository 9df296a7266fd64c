"""Pins for the oracle's router and permutation (CPU only).

Top-k is checked against an exhaustive Python sort of (-logit, expert)
tuples; the weights against closed forms; the permutation against its
defining invariants and a brute-force stable placement.
"""

import itertools

import numpy as np
import pytest

import oracle


def _brute_topk(row, k):
    # Exhaustive: order every expert by (-logit, index) with Python's sort.
    order = sorted(range(len(row)), key=lambda e: (-float(row[e]), e))
    return order[:k]


@pytest.mark.parametrize("E", [1, 2, 3, 5, 6])
def test_topk_matches_exhaustive_sort(E):
    rng = np.random.default_rng(E)
    for k in range(1, E + 1):
        for trial in range(6):
            logits = rng.standard_normal((4, E)).astype(np.float32)
            if trial % 2:
                logits = np.round(logits)  # many duplicates -> tie-break
            idx, _ = oracle.route_topk(logits, k)
            for t in range(4):
                assert list(idx[t]) == _brute_topk(logits[t], k)


def test_topk_by_subset_enumeration():
    # The chosen set maximises the sum of logits over all k-subsets (distinct
    # logits so the maximiser is unique).
    rng = np.random.default_rng(7)
    logits = rng.permutation(np.arange(6, dtype=np.float32))[None, :] * 0.37
    for k in range(1, 7):
        idx, _ = oracle.route_topk(logits, k)
        best = max(itertools.combinations(range(6), k),
                   key=lambda s: sum(float(logits[0, e]) for e in s))
        assert set(idx[0].tolist()) == set(best)


def test_ties_lower_expert_first():
    logits = np.array([[0.5, 1.0, 1.0, 0.5, 1.0]], dtype=np.float32)
    idx, w = oracle.route_topk(logits, 4)
    assert list(idx[0]) == [1, 2, 4, 0]
    assert np.allclose(w[0, :3], w[0, 0])


def test_weights_closed_forms():
    T, E, k = 5, 8, 3
    flat = np.zeros((T, E), dtype=np.float32)
    _, w = oracle.route_topk(flat, k, renormalize=True)
    assert np.allclose(w, 1.0 / k, rtol=0, atol=1e-15)
    _, w = oracle.route_topk(flat, k, renormalize=False)
    assert np.allclose(w, 1.0 / E, rtol=0, atol=1e-15)
    # Two experts, k = 1, logit gap d: the winner's probability is sigmoid(d).
    d = 0.75
    _, w = oracle.route_topk(np.array([[d, 0.0]], np.float32), 1, renormalize=False)
    assert abs(w[0, 0] - 1 / (1 + np.exp(-d))) < 1e-15


def test_renormalised_weights_sum_to_one_and_equal_local_softmax():
    rng = np.random.default_rng(11)
    logits = (rng.standard_normal((64, 128)) * 3).astype(np.float32)
    idx, w = oracle.route_topk(logits, 8, renormalize=True)
    assert np.allclose(w.sum(1), 1.0, atol=1e-12)
    sel = np.take_along_axis(logits.astype(np.float64), idx.astype(np.int64), 1)
    local = np.exp(sel - sel.max(1, keepdims=True))
    local /= local.sum(1, keepdims=True)
    assert np.allclose(w, local, rtol=1e-12, atol=1e-15)
    assert np.all(np.diff(w, axis=1) <= 1e-15), "weights follow descending logits"
    _, w2 = oracle.route_topk(logits, 8, renormalize=False)
    assert np.all(w2.sum(1) <= 1 + 1e-12)


def _check_permutation(idx, E, offsets, sorted_rows, inv_perm):
    flat = idx.reshape(-1)
    n = flat.size
    assert offsets[0] == 0 and offsets[-1] == n
    assert np.all(np.diff(offsets) >= 0)
    assert np.array_equal(np.diff(offsets), np.bincount(flat, minlength=E))
    assert np.array_equal(np.sort(sorted_rows), np.arange(n))
    experts = flat[sorted_rows]
    assert np.all(np.diff(experts) >= 0)
    for e in range(E):
        seg = sorted_rows[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e)
        assert np.all(np.diff(seg) > 0), "stable: flat ids ascend in a segment"
    assert np.array_equal(inv_perm[sorted_rows], np.arange(n))


@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (16, 8, 2), (37, 64, 8), (5, 4, 4), (0, 8, 2)])
def test_permutation_invariants(T, E, k):
    rng = np.random.default_rng(T * 100 + E)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    idx, _ = oracle.route_topk(logits, k) if T else (np.zeros((0, k), np.int32), None)
    offsets, sorted_rows, inv_perm = oracle.permute_by_expert(idx, E)
    _check_permutation(idx, E, offsets, sorted_rows, inv_perm)


def test_permutation_brute_force_placement():
    # Place flat ids one expert at a time, scanning in flat order.
    rng = np.random.default_rng(5)
    idx = rng.integers(0, 6, size=(9, 3)).astype(np.int32)
    flat = idx.reshape(-1).tolist()
    brute = [f for e in range(6) for f in range(len(flat)) if flat[f] == e]
    _, sorted_rows, _ = oracle.permute_by_expert(idx, 6)
    assert sorted_rows.tolist() == brute


def test_permutation_gate_catches_a_swap():
    # Planted mistake: swapping two positions of different experts breaks the
    # invariants the GPU result is also held to.
    rng = np.random.default_rng(9)
    idx = rng.integers(0, 5, size=(7, 2)).astype(np.int32)
    offsets, sorted_rows, inv_perm = oracle.permute_by_expert(idx, 5)
    bad = sorted_rows.copy()
    p = int(offsets[1]) - 1 if offsets[1] > 0 else 0
    q = int(offsets[-1]) - 1
    bad[p], bad[q] = bad[q], bad[p]
    with pytest.raises(AssertionError):
        _check_permutation(idx, 5, offsets, bad, inv_perm)
