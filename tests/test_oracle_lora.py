"""Pins for the per-expert LoRA delta oracle (``oracle.lora``).

The definition fixes: the delta of a routed row is scale * B_e A_e x; summed
with the frozen product it equals the product with the merged weight
W_e + scale * B_e A_e; the merged update has rank at most r; and it is linear
in scale and zero when B_e is zero (LoRA's initialisation)."""

import numpy as np

import oracle


def _setup(seed=0, E=3, N=24, K=32, r=4, counts=(2, 0, 3)):
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((E, r, K))
    B = rng.standard_normal((E, N, r))
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    X = rng.standard_normal((int(off[-1]), K))
    return rng, A, B, off, X


def test_equals_merged_weight_product():
    rng, A, B, off, X = _setup()
    W = rng.standard_normal((3, 24, 32))
    scale = 0.5
    d = oracle.lora_delta(X, off, A, B, scale)
    for e in range(3):
        Wm = W[e] + scale * B[e] @ A[e]          # merged (dense) adapter
        for p in range(off[e], off[e + 1]):
            np.testing.assert_allclose(W[e] @ X[p] + d[p], Wm @ X[p], rtol=1e-12, atol=1e-12)


def test_update_has_rank_at_most_r():
    _, A, B, off, _ = _setup(r=4)
    for e in range(3):
        # the delta map x -> delta is B_e A_e: probe it with the identity
        M = oracle.lora_delta(np.eye(32), np.array([0, 32]), A[e:e + 1], B[e:e + 1], 1.0)
        assert np.linalg.matrix_rank(M) <= 4
        np.testing.assert_allclose(M.T, B[e] @ A[e], rtol=1e-12, atol=1e-12)


def test_linear_in_scale_and_zero_for_zero_b():
    _, A, B, off, X = _setup()
    d1 = oracle.lora_delta(X, off, A, B, 1.0)
    np.testing.assert_allclose(oracle.lora_delta(X, off, A, B, -2.5), -2.5 * d1, rtol=1e-12)
    assert not np.any(oracle.lora_delta(X, off, A, np.zeros_like(B), 1.0))


def test_rows_subset_and_segments():
    _, A, B, off, X = _setup()
    full = oracle.lora_delta(X, off, A, B, 0.25)
    np.testing.assert_array_equal(oracle.lora_delta(X, off, A, B, 0.25, rows=[4, 0]), full[[4, 0]])
    # row 2 belongs to expert 2 (expert 1 is empty): swapping expert 2's
    # adapters changes it, expert 0's rows stay
    B2 = B.copy()
    B2[2] *= 3
    alt = oracle.lora_delta(X, off, A, B2, 0.25)
    np.testing.assert_allclose(alt[2:], 3 * full[2:], rtol=1e-12)
    np.testing.assert_array_equal(alt[:2], full[:2])
