"""Pins for the grouped INT4 oracle (``oracle.int4``).

The pages name the format only as GPTQ-calibrated int4; the readings (group
of 128 along K, fp16 scale, 4-bit zero, w = (q - z) * s, range containing 0,
round to nearest even) are stated in ``oracle/int4.py``.  These tests pin the
oracle to what that definition fixes independently of its code: exact
recovery of values on the grid, the rounding error bound, brute-force
nearest-grid agreement, group independence, the byte layout, and the
grouped GEMM against a plain per-expert matmul.
"""

import numpy as np
import pytest

import oracle

G = oracle.INT4_GROUP


def _grid_values(rng, rows, groups):
    """Weights that lie exactly on a grid (q - z) * s with both ends of the
    code range present in every group, so the definition must recover them."""
    s = rng.uniform(1e-3, 5e-2, size=(rows, groups)).astype(np.float16)
    z = rng.integers(0, 16, size=(rows, groups))
    q = rng.integers(0, 16, size=(rows, groups, G))
    q[..., 0] = 0
    q[..., 1] = 15
    x = ((q - z[..., None]) * s[..., None].astype(np.float64)).astype(np.float32)
    return x.reshape(rows, groups * G), q.reshape(rows, groups * G), s, z


def test_grid_values_recovered_exactly():
    rng = np.random.default_rng(0)
    x, q, s, z = _grid_values(rng, 6, 3)
    packed, meta = oracle.quantize_int4_grouped(x)
    s2, z2 = oracle.int4_scales_zeros(meta)
    assert np.array_equal(s2, s.astype(np.float32))
    assert np.array_equal(z2, z)
    codes = np.empty_like(q)
    codes[:, 0::2] = packed >> 4
    codes[:, 1::2] = packed & 15
    assert np.array_equal(codes, q)
    assert np.array_equal(oracle.dequantize_int4_grouped(packed, meta), x.astype(np.float64))


def test_byte_layout_and_meta_bits():
    # one row, one group: codes 0..15 repeated; grid s = 0.5, z = 3
    q = np.tile(np.arange(16), G // 16)
    x = ((q - 3) * 0.5).astype(np.float32)[None]
    packed, meta = oracle.quantize_int4_grouped(x)
    assert packed.shape == (1, G // 2) and meta.shape == (1, 1)
    assert list(packed[0, :3]) == [0x01, 0x23, 0x45]    # even element in the high nibble
    assert int(meta[0, 0]) == (0x3800 | (3 << 16))       # fp16(0.5) = 0x3800, zero 3


def test_all_zero_group():
    x = np.zeros((2, 2 * G), np.float32)
    x[1, G:] = np.linspace(-1, 1, G)
    packed, meta = oracle.quantize_int4_grouped(x)
    assert np.all(meta[0] == 0) and np.all(packed[0] == 0) and meta[1, 0] == 0
    w = oracle.dequantize_int4_grouped(packed, meta)
    assert np.all(w[0] == 0) and np.all(w[1, :G] == 0)


def test_error_bound_and_nearest_grid_point():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((64, 4 * G)) * 0.02).astype(np.float32)
    x[rng.random(x.shape) < 1e-3] *= 8.0                  # outliers widen some groups
    packed, meta = oracle.quantize_int4_grouped(x)
    w = oracle.dequantize_int4_grouped(packed, meta)
    s, z = oracle.int4_scales_zeros(meta)
    s_e = np.repeat(s, G, axis=1).astype(np.float64)
    z_e = np.repeat(z, G, axis=1)
    err = np.abs(x - w)
    # one grid step at most (half a step plus the fp16 rounding of s and the
    # rounding of the zero point), half a step away from the clamped ends
    assert np.all(err <= 1.01 * s_e)
    # brute force: the chosen code is the grid point nearest to x, clamped
    cand = (np.arange(16)[None, None, :] - z_e[..., None]) * s_e[..., None]
    best = np.argmin(np.abs(x[..., None] - cand), axis=-1)
    codes = np.empty_like(best)
    codes[:, 0::2] = packed >> 4
    codes[:, 1::2] = packed & 15
    dis = codes != best
    # disagreements only where two grid points are (almost) equally near
    d1 = np.abs(x - (codes - z_e) * s_e)
    d2 = np.abs(x - (best - z_e) * s_e)
    assert dis.mean() < 1e-3
    assert np.all(np.abs(d1[dis] - d2[dis]) <= 1e-6 * s_e[dis])


def test_groups_are_independent_and_128_wide():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((3, 3 * G)) * 0.02).astype(np.float32)
    p1, m1 = oracle.quantize_int4_grouped(x)
    y = x.copy()
    y[:, G + 5] = 3.0                                     # only the middle group changes
    p2, m2 = oracle.quantize_int4_grouped(y)
    assert np.array_equal(m1[:, [0, 2]], m2[:, [0, 2]])
    assert not np.array_equal(m1[:, 1], m2[:, 1])
    assert np.array_equal(p1[:, : G // 2], p2[:, : G // 2])
    assert np.array_equal(p1[:, G:], p2[:, G:])


def test_planted_mistakes_fail():
    # a symmetric quantizer (zero fixed at 8) misses grid values the
    # definition recovers exactly
    rng = np.random.default_rng(3)
    x, q, s, z = _grid_values(rng, 4, 2)
    sym = np.clip(np.rint(x.reshape(4, 2, G) / s[..., None].astype(np.float32)) + 8, 0, 15)
    assert not np.array_equal(sym.reshape(q.shape), q)
    # truncating instead of rounding fails the nearest-grid check the oracle
    # passes (same scales and zeros, so only the rounding rule differs)
    y = (rng.standard_normal((8, 2 * G)) * 0.02).astype(np.float32)
    packed, meta = oracle.quantize_int4_grouped(y)
    s2, z2 = oracle.int4_scales_zeros(meta)
    s_e = np.repeat(s2, G, axis=1)
    z_e = np.repeat(z2, G, axis=1)
    trunc = np.clip(np.trunc(y / s_e) + z_e, 0, 15)
    cand = (np.arange(16)[None, None, :] - z_e[..., None]) * s_e[..., None].astype(np.float64)
    best = np.argmin(np.abs(y[..., None] - cand), axis=-1)
    assert (trunc != best).mean() > 0.2


def test_grouped_gemm_int4_matches_per_expert_matmul():
    rng = np.random.default_rng(4)
    E, N, K = 3, 8, 2 * G
    W = (rng.standard_normal((E, N, K)) * 0.05).astype(np.float32)
    packed, meta = oracle.quantize_int4_grouped(W)
    counts = [2, 0, 3]
    off = np.concatenate([[0], np.cumsum(counts)])
    A = rng.standard_normal((off[-1], K))
    out = oracle.grouped_gemm_int4(A, packed, meta, off)
    for e in range(E):
        Wd = oracle.dequantize_int4_grouped(packed[e], meta[e])
        for p in range(off[e], off[e + 1]):
            np.testing.assert_allclose(out[p], Wd @ A[p], rtol=1e-12, atol=1e-12)


def test_rejects_k_not_multiple_of_group():
    with pytest.raises(ValueError):
        oracle.quantize_int4_grouped(np.zeros((1, 64), np.float32))


def test_int4_layer_equals_dense_brute_force():
    # the routed layer on INT4 experts equals the all-experts-dense form
    rng = np.random.default_rng(5)
    E, k, H, I, T = 4, 2, 256, 128, 5
    w_gu = (rng.standard_normal((E, 2 * I, H)) * 0.05).astype(np.float32)
    w_d = (rng.standard_normal((E, H, I)) * 0.05).astype(np.float32)
    p_gu, m_gu = oracle.quantize_int4_grouped(w_gu)
    p_d, m_d = oracle.quantize_int4_grouped(w_d)
    stack = oracle.Int4ExpertStack(p_gu, m_gu, p_d, m_d)
    x = rng.standard_normal((T, H)).astype(np.float32)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    y = oracle.moe_layer(x, lg, stack, k, True)
    y_dense = oracle.moe_layer_dense(x, lg, stack, k, True)
    np.testing.assert_allclose(y, y_dense, rtol=1e-9, atol=1e-12)
