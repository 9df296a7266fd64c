"""Pins for the oracle's NF4 quantizer (CPU only).

Each test ties ``oracle.nf4`` to something other than itself: the published
QLoRA table, the quantile construction recomputed with two inverse-normal
routines, closed forms (exact levels, zero blocks), brute-force nearest level,
the error bound of a nearest-level quantizer, idempotence, and the byte
totals the pages print.  The planted-mistake tests show each gate can fail.
"""

import os
import statistics

import numpy as np
import pytest
from scipy.stats import norm

import oracle
from oracle import nf4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line)
    return rows


def test_levels_match_published_table():
    pub = np.array([float(r) for r in _read_golden("nf4_levels_qlora.txt")],
                   dtype=np.float32)
    assert pub.size == 16
    assert np.array_equal(oracle.nf4_levels().view(np.int32), pub.view(np.int32))


def test_levels_structure():
    L = oracle.nf4_levels()
    assert L.dtype == np.float32 and L.size == 16
    assert np.all(np.diff(L) > 0), "strictly ascending"
    assert L[0] == -1.0 and L[7] == 0.0 and L[15] == 1.0
    assert (L < 0).sum() == 7 and (L == 0).sum() == 1 and (L > 0).sum() == 8
    # "symmetric in spirit": every negative magnitude lies inside the range of
    # the positive magnitudes, and the levels are centred near zero.
    pos = L[L > 0]
    for m in -L[L < 0]:
        assert pos.min() <= m <= pos.max()
    assert abs(float(L.astype(np.float64).mean())) < 0.1


@pytest.mark.parametrize("inv_cdf", [norm.ppf, statistics.NormalDist().inv_cdf],
                         ids=["scipy", "statistics"])
def test_levels_follow_quantile_construction(inv_cdf):
    v = oracle.nf4_levels_from_quantiles(inv_cdf)
    # The published fp32 table was rounded through float32 intermediates; it
    # agrees with the exact construction to a few fp32 ulps.
    assert np.max(np.abs(v - oracle.nf4_levels().astype(np.float64))) < 1e-6


def test_two_quantile_routines_agree():
    a = oracle.nf4_levels_from_quantiles(norm.ppf)
    b = oracle.nf4_levels_from_quantiles(statistics.NormalDist().inv_cdf)
    assert np.max(np.abs(a - b)) < 1e-12


def test_construction_pin_fails_on_a_wrong_offset():
    # Planted mistake: the textbook construction with the outer quantile at
    # 0.99 instead of delta must not pass the table pin.
    delta = 0.99
    pos = norm.ppf(np.linspace(delta, 0.5, 9)[:-1])
    neg = -norm.ppf(np.linspace(delta, 0.5, 8)[:-1])
    v = np.sort(np.concatenate([neg, [0.0], pos]))
    v /= np.abs(v).max()
    assert np.max(np.abs(v - oracle.nf4_levels())) > 1e-3


def test_midpoints_lie_between_levels():
    L = oracle.nf4_levels()
    M = oracle.nf4_midpoints()
    assert M.dtype == np.float32 and M.size == 15
    assert np.all(L[:-1] < M) and np.all(M < L[1:])


def test_exact_levels_quantize_to_their_codes_and_pack_high_nibble_first():
    # Closed form: a block whose elements are exactly a * L[c] has absmax a
    # (the code-0 or code-15 element) and quantizes to c everywhere.
    rng = np.random.default_rng(1)
    codes = rng.integers(0, 16, size=64).astype(np.uint8)
    codes[5] = 15
    a = np.float32(2.0)  # power of two: a * L[c] / a == L[c] exactly
    x = (oracle.nf4_levels()[codes] * a).astype(np.float32)[None, :]
    packed, absmax = oracle.quantize_blockwise(x)
    assert absmax.shape == (1, 1) and absmax[0, 0] == a
    expect = bytes(int(codes[2 * j]) * 16 + int(codes[2 * j + 1]) for j in range(32))
    assert packed.tobytes() == expect


def test_hand_example_bytes():
    # Hand-derived: x = [2, -2, 0, 1.1245940, ...zeros]; absmax 2, n = [1, -1,
    # 0, 0.5622970]; 0.5623 lies between midpoints M_12 = 0.5017 and
    # M_13 = 0.6428 -> code 13.  Bytes: (15<<4)|0 = 0xF0, (7<<4)|13 = 0x7D,
    # then 0x77 for the zero pairs.
    x = np.zeros((1, 64), dtype=np.float32)
    x[0, :4] = [2.0, -2.0, 0.0, 1.124594]
    packed, absmax = oracle.quantize_blockwise(x)
    assert absmax[0, 0] == 2.0
    assert packed[0, 0] == 0xF0 and packed[0, 1] == 0x7D
    assert np.all(packed[0, 2:] == 0x77)


def test_swapped_nibble_order_fails_hand_example():
    # Planted mistake: low nibble first would give 0x0F for the first byte.
    x = np.zeros((1, 64), dtype=np.float32)
    x[0, :2] = [2.0, -2.0]
    packed, _ = oracle.quantize_blockwise(x)
    c = oracle.unpack_codes(packed)
    wrong = (c[0, 1] << 4) | c[0, 0]
    assert wrong != packed[0, 0]


def test_zero_block():
    x = np.zeros((2, 128), dtype=np.float32)
    x[1, 64:] = np.linspace(-1, 1, 64, dtype=np.float32)
    packed, absmax = oracle.quantize_blockwise(x)
    assert absmax[0, 0] == 0 and absmax[0, 1] == 0 and absmax[1, 0] == 0
    assert np.all(oracle.unpack_codes(packed)[:, :64] == 7)
    assert np.all(oracle.unpack_codes(packed)[0] == 7)
    w = oracle.dequantize_blockwise(packed, absmax)
    assert np.all(w[0] == 0) and np.all(w[1, :64] == 0)


def test_nearest_level_brute_force():
    # For normalised values away from a midpoint, the code is the argmin of
    # |n - L_i| computed in fp64.
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 64)).astype(np.float32)
    packed, absmax = oracle.quantize_blockwise(x)
    codes = oracle.unpack_codes(packed).reshape(-1)
    n = (x / absmax).astype(np.float64).reshape(-1)
    L = oracle.nf4_levels().astype(np.float64)
    brute = np.argmin(np.abs(n[:, None] - L[None, :]), axis=1)
    M = oracle.nf4_midpoints().astype(np.float64)
    near_mid = np.min(np.abs(n[:, None] - M[None, :]), axis=1) < 1e-6
    assert np.all((codes == brute) | near_mid)
    assert near_mid.sum() < 3


def test_ties_go_to_lower_code():
    M = oracle.nf4_midpoints()
    x = np.zeros((1, 64), dtype=np.float32)
    x[0, 0] = 1.0          # absmax 1, so n == x exactly
    x[0, 1:16] = M         # exactly on each midpoint
    codes = oracle.unpack_codes(oracle.quantize_blockwise(x)[0])[0]
    assert list(codes[1:16]) == list(range(15))


def test_roundtrip_error_bound_and_idempotence():
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((3, 16, 256)) * 0.02).astype(np.float32)
    W[0, 0, 10] = 0.16  # an 8-sigma outlier
    packed, absmax = oracle.quantize_blockwise(W)
    D = oracle.dequantize_blockwise(packed, absmax)
    L = oracle.nf4_levels().astype(np.float64)
    half_gap = np.max(np.diff(L)) / 2
    a = np.repeat(absmax.astype(np.float64), 64, axis=-1)
    assert np.all(np.abs(W - D) <= a * half_gap * (1 + 1e-6))
    # Q(D(Q(W))) == Q(W) bit for bit: every dequantized value sits on a level
    # and the block maximum dequantizes to +-absmax exactly.
    p2, a2 = oracle.quantize_blockwise(D.astype(np.float32))
    assert np.array_equal(p2, packed)
    assert np.array_equal(a2.view(np.int32), absmax.view(np.int32))


def test_idempotence_gate_catches_a_flipped_nibble():
    # Planted mistake: flip one nibble of the packed codes; the round trip of
    # the corrupted codes no longer reproduces the original bytes.
    rng = np.random.default_rng(4)
    W = rng.standard_normal((4, 128)).astype(np.float32)
    packed, absmax = oracle.quantize_blockwise(W)
    bad = packed.copy()
    bad[1, 3] ^= 0x10
    p2, _ = oracle.quantize_blockwise(oracle.dequantize_blockwise(bad, absmax).astype(np.float32))
    assert not np.array_equal(p2, packed)


def test_nonfinite_rejected():
    x = np.zeros((1, 64), dtype=np.float32)
    x[0, 3] = np.inf
    with pytest.raises(ValueError):
        oracle.quantize_blockwise(x)


@pytest.mark.parametrize("blocksize,absmax_bytes,should_match", [
    (64, 4, True),      # the reading taken: blocksize 64, fp32 absmax
    (64, 2, False),     # fp16 absmax
    (32, 4, False),     # smaller blocks
    (128, 4, False),    # larger blocks
])
def test_page_byte_totals_pin_block_geometry(blocksize, absmax_bytes, should_match):
    for row in _read_golden("page_byte_totals.txt"):
        name, layers, E, H, I, total, _src = row.split()
        n = 3 * int(H) * int(I)
        per_expert = n // 2 + (n // blocksize) * absmax_bytes
        got = int(layers) * int(E) * per_expert
        rel = abs(got - float(total)) / float(total)
        # "16.31 GB" is quoted to 4 digits, "about 128 GB" to 3.
        tol = 5e-4 if name == "qwen3-30b-a3b" else 5e-3
        assert (rel < tol) == should_match, (name, got, total)
