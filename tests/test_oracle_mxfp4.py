"""Pins for the MXFP4 oracle (``oracle.mxfp4``).

The format is fixed by the OCP Microscaling v1.0 definitions the pages name
(e2m1 elements, e8m0 scales).  These tests pin the oracle to what those
definitions fix independently of its code: the E2M1 values decoded from their
bit fields, exact recovery of on-grid blocks, round-to-nearest-even at every
midpoint, saturation, brute-force nearest-value agreement, the shared
exponent rule, the byte layout, and the grouped GEMM against a per-expert
matmul.
"""

import numpy as np
import pytest

import oracle

B = oracle.MXFP4_BLOCK


def test_e2m1_values_from_bit_fields():
    # sign | 2-bit exponent (bias 1) | 1-bit mantissa; exponent 0 is subnormal
    got = oracle.e2m1_values()
    for c in range(16):
        s, e, m = c >> 3, (c >> 1) & 3, c & 1
        mag = 0.5 * m if e == 0 else 2.0 ** (e - 1) * (1 + 0.5 * m)
        assert got[c] == (-mag if s else mag)
        assert np.signbit(got[c]) == bool(s)


def _codes(packed):
    c = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.int64)
    c[..., 0::2] = packed & 15
    c[..., 1::2] = packed >> 4
    return c


def test_on_grid_blocks_are_recovered_exactly():
    rng = np.random.default_rng(0)
    vals = oracle.e2m1_values()
    codes = rng.integers(0, 16, size=(5, 4 * B))
    s = rng.integers(-20, 5, size=(5, 4))
    x = (vals[codes].reshape(5, 4, B) * np.exp2(s)[..., None]).reshape(5, 4 * B)
    x = x.astype(np.float32)
    packed, scales = oracle.quantize_mxfp4(x)
    w = oracle.dequantize_mxfp4(packed, scales)
    assert np.array_equal(w, x.astype(np.float64))
    # the stored block is normalised: its largest code magnitude is 4 or 6
    mags = np.abs(vals[_codes(packed)]).reshape(5, 4, B).max(axis=-1)
    nz = np.abs(x).reshape(5, 4, B).max(axis=-1) > 0
    assert np.all(np.isin(mags[nz], [4.0, 6.0]))


def test_round_to_nearest_even_at_midpoints_and_saturation():
    # amax = 6 -> shared exponent floor(log2 6) - 2 = 0, so y = x
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    want = [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]
    x = np.zeros((1, B), np.float32)
    x[0, 0] = 6.0
    x[0, 1:8] = mids
    x[0, 8:15] = [-m for m in mids]
    x[0, 15] = 0.26                         # just above a midpoint
    packed, scales = oracle.quantize_mxfp4(x)
    w = oracle.dequantize_mxfp4(packed, scales)[0]
    assert scales[0, 0] == 127
    assert list(w[1:8]) == want
    assert list(w[8:15]) == [-v for v in want]
    assert w[15] == 0.5
    # amax = 7 keeps exponent 0 (floor(log2 7) = 2) and saturates 7 to 6
    y = np.zeros((1, B), np.float32)
    y[0, 0], y[0, 1] = 7.0, -7.0
    p2, s2 = oracle.quantize_mxfp4(y)
    w2 = oracle.dequantize_mxfp4(p2, s2)[0]
    assert s2[0, 0] == 127 and w2[0] == 6.0 and w2[1] == -6.0


def test_codes_are_the_nearest_values_brute_force():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((16, 8 * B)) * 0.02).astype(np.float32)
    x[rng.random(x.shape) < 2e-3] *= 10.0
    packed, scales = oracle.quantize_mxfp4(x)
    codes = _codes(packed).reshape(16, 8, B)
    # the shared exponent rule, from the definition
    amax = np.abs(x).reshape(16, 8, B).max(axis=-1)
    assert np.array_equal(scales.astype(np.int64) - 127, np.floor(np.log2(amax)).astype(int) - 2)
    y = x.reshape(16, 8, B).astype(np.float64) / np.exp2(scales.astype(np.float64) - 127)[..., None]
    vals = oracle.e2m1_values()
    d = np.abs(np.clip(y, -6, 6)[..., None] - vals)
    chosen = np.take_along_axis(d, codes[..., None], axis=-1)[..., 0]
    assert np.all(chosen <= d.min(axis=-1))
    # saturation is the only way to be more than half a step away
    err = np.abs(x - oracle.dequantize_mxfp4(packed, scales))
    step = np.exp2(scales.astype(np.float64) - 127)      # E2M1 spacing is <= 2 x 2^shared
    assert np.all(err.reshape(16, 8, B) <= np.maximum(1.0 * step[..., None],
                                                       np.abs(x.reshape(16, 8, B)) - 6 * step[..., None]))


def test_byte_layout_and_scale_byte():
    x = np.zeros((1, B), np.float32)
    x[0, :4] = [1.0, -0.5, 6.0, 0.0]
    packed, scales = oracle.quantize_mxfp4(x)
    assert scales.shape == (1, 1) and packed.shape == (1, B // 2)
    assert int(scales[0, 0]) == 127                       # 2^0
    assert list(packed[0, :2]) == [0x92, 0x07]            # element 2j in the low nibble
    # a block scaled by 2^-10 stores 117
    p2, s2 = oracle.quantize_mxfp4(x * np.float32(2 ** -10))
    assert int(s2[0, 0]) == 117 and np.array_equal(p2, packed)


def test_zero_and_tiny_blocks():
    x = np.zeros((2, 2 * B), np.float32)
    x[1, B] = np.float32(2.0 ** -130)                      # fp32 subnormal
    packed, scales = oracle.quantize_mxfp4(x)
    assert np.all(packed[0] == 0) and np.all(scales[0] == 0)
    # the shared exponent clamps at -127 (scale byte 0): 2^-130 = 2^-127 * 0.125
    # rounds to 0 (the nearest E2M1 value to 0.125)
    assert scales[1, 1] == 0
    assert np.all(oracle.dequantize_mxfp4(packed, scales) == 0)


def test_rejects_bad_input():
    with pytest.raises(ValueError):
        oracle.quantize_mxfp4(np.zeros((1, 48), np.float32))
    with pytest.raises(ValueError):
        oracle.quantize_mxfp4(np.full((1, 32), np.inf, np.float32))
    with pytest.raises(ValueError):
        oracle.dequantize_mxfp4(np.zeros((1, 16), np.uint8), np.full((1, 1), 255, np.uint8))


def test_planted_mistakes_fail():
    rng = np.random.default_rng(2)
    vals = oracle.e2m1_values()
    codes = rng.integers(0, 16, size=(4, 2 * B))
    x = (vals[codes] * 2.0 ** -6).astype(np.float32)
    packed, scales = oracle.quantize_mxfp4(x)
    # high-nibble-first unpacking (NF4's order) scrambles on-grid values
    c = np.empty((4, 2 * B), np.int64)
    c[:, 0::2] = packed >> 4
    c[:, 1::2] = packed & 15
    wrong = vals[c].reshape(4, 2, B) * np.exp2(scales.astype(np.float64) - 127)[..., None]
    assert not np.array_equal(wrong.reshape(4, 2 * B), x.astype(np.float64))
    # a ceil(log2 amax) - 2 exponent rule (instead of floor) halves the block
    # before rounding, so 1.5 -> 0.75 -> 1.0 and on-grid values are lost
    y = np.array([6.0, 1.5, 0.5, 3.0])
    sh = int(np.ceil(np.log2(6.0))) - 2
    near = vals[np.argmin(np.abs((y / 2.0 ** sh)[:, None] - vals), axis=1)] * 2.0 ** sh
    assert not np.array_equal(near, y)
    z = np.zeros((1, B), np.float32)
    z[0, :4] = y
    assert np.array_equal(oracle.dequantize_mxfp4(*oracle.quantize_mxfp4(z))[0, :4], y)


def test_grouped_gemm_mxfp4_matches_per_expert_matmul():
    rng = np.random.default_rng(3)
    E, N, K = 3, 8, 4 * B
    W = (rng.standard_normal((E, N, K)) * 0.05).astype(np.float32)
    packed, scales = oracle.quantize_mxfp4(W)
    counts = [2, 0, 3]
    off = np.concatenate([[0], np.cumsum(counts)])
    A = rng.standard_normal((off[-1], K))
    out = oracle.grouped_gemm_mxfp4(A, packed, scales, off)
    for e in range(E):
        Wd = oracle.dequantize_mxfp4(packed[e], scales[e])
        for p in range(off[e], off[e + 1]):
            np.testing.assert_allclose(out[p], Wd @ A[p], rtol=1e-12, atol=1e-12)


def test_mxfp4_layer_equals_dense_brute_force():
    rng = np.random.default_rng(4)
    E, k, H, I, T = 4, 2, 64, 64, 5
    w_gu = (rng.standard_normal((E, 2 * I, H)) * 0.05).astype(np.float32)
    w_d = (rng.standard_normal((E, H, I)) * 0.05).astype(np.float32)
    stack = oracle.Mxfp4ExpertStack(*oracle.quantize_mxfp4(w_gu), *oracle.quantize_mxfp4(w_d))
    x = rng.standard_normal((T, H)).astype(np.float32)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    y = oracle.moe_layer(x, lg, stack, k, True)
    np.testing.assert_allclose(y, oracle.moe_layer_dense(x, lg, stack, k, True), rtol=1e-9,
                               atol=1e-12)
