"""NF4 blockwise quantize / dequantize, written out from its definition.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What the pages fix ("grouped-nf4-gemm & experts-4bit", jordananderson-pages
.pages.dev, first and third bullets): a sixteen-entry NF4 codebook on the
bitsandbytes packed layout, two 4-bit codes per byte and a per-block absmax.
The problem statement fixes blocksize 64 and an fp32 absmax with no nested
quantization.  The pages print neither the level values, the nibble order
nor the rounding rule; the readings taken here are:

* levels: the NF4 codebook as published with QLoRA (Dettmers et al., 2023,
  appendix "NormalFloat 4-bit data type"), i.e. the bitsandbytes table, in
  fp32.  It is pinned in the tests against the quantile construction the
  QLoRA paper defines (recomputed here with two independent inverse-normal
  routines) to within 1e-6;
* blocks: 64 consecutive elements of each expert's row-major [N, K] matrix;
  since K % 64 == 0 they run along K, the reduction dimension;
* normalisation: n = x / absmax in IEEE fp32 (correctly rounded division);
* code: the number of fp32 midpoints M_i = fl32(L_i + L_{i+1}) * 0.5 that n
  lies strictly above -- the nearest level, ties going to the lower code;
* an all-zero block gets absmax 0 and every code 7 (the level 0.0);
* packing: element 2j of a row goes to the HIGH nibble of byte j, element
  2j+1 to the low nibble (bitsandbytes' order);
* dequantize: w = L[code] * absmax.  Both factors are fp32, so the product
  is exact in fp64, which is what ``dequantize_blockwise`` returns.
"""

from __future__ import annotations

import numpy as np

BLOCKSIZE = 64

# The sixteen NF4 levels as published with QLoRA (appendix table of the
# NormalFloat data type), ascending.  Code 7 is exactly 0, codes 0 and 15
# are exactly -1 and +1.
_NF4_PUBLISHED = (
    -1.0,
    -0.6961928009986877,
    -0.5250730514526367,
    -0.39491748809814453,
    -0.28444138169288635,
    -0.18477343022823334,
    -0.09105003625154495,
    0.0,
    0.07958029955625534,
    0.16093020141124725,
    0.24611230194568634,
    0.33791524171829224,
    0.44070982933044434,
    0.5626170039176941,
    0.7229568362236023,
    1.0,
)


def nf4_levels() -> np.ndarray:
    """The 16 NF4 levels as float32, ascending (code c -> level c)."""
    return np.array(_NF4_PUBLISHED, dtype=np.float32)


def nf4_levels_from_quantiles(inv_cdf) -> np.ndarray:
    """NF4 levels rebuilt from the QLoRA quantile construction, in fp64.

    The construction: take the standard-normal quantiles at 8 equally spaced
    probabilities from delta down to 1/2 (exclusive) for the positive side and
    at 7 for the negative side, where delta = 1 - (1/(2*15) + 1/(2*16)) / 2
    keeps the outermost quantile finite; add one exact zero; sort; divide by
    the largest magnitude so the ends are exactly -1 and +1.

    ``inv_cdf`` maps a probability to a standard-normal quantile; the tests
    pass two independent implementations.  Used only to pin ``nf4_levels``.
    """
    delta = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0)
    p_pos = np.linspace(delta, 0.5, 9)[:-1]
    p_neg = np.linspace(delta, 0.5, 8)[:-1]
    pos = np.array([inv_cdf(float(p)) for p in p_pos], dtype=np.float64)
    neg = -np.array([inv_cdf(float(p)) for p in p_neg], dtype=np.float64)
    v = np.sort(np.concatenate([neg, [0.0], pos]))
    return v / np.max(np.abs(v))


def nf4_midpoints(levels: np.ndarray | None = None) -> np.ndarray:
    """The 15 fp32 decision thresholds fl32(L_i + L_{i+1}) * 0.5."""
    L = nf4_levels() if levels is None else np.asarray(levels, dtype=np.float32)
    s = (L[:-1] + L[1:]).astype(np.float32)  # fp32 add, one rounding
    return (s * np.float32(0.5)).astype(np.float32)  # exact halving


def quantize_blockwise(W: np.ndarray, blocksize: int = BLOCKSIZE):
    """Quantize ``W[..., K]`` (float32) to NF4 with one fp32 absmax per block.

    Returns ``(packed uint8[..., K/2], absmax float32[..., K/blocksize])``.
    For the fused expert stack ``W[E, N, K]`` the absmax array is the
    row-major ``[E, N*K/64]`` of the library's layout.
    """
    W = np.asarray(W)
    if W.dtype != np.float32:
        raise TypeError("quantize_blockwise expects float32 weights")
    if blocksize != BLOCKSIZE:
        raise ValueError("only blocksize 64 is defined")
    K = W.shape[-1]
    if K % blocksize:
        raise ValueError("K must be a multiple of the blocksize")
    if not np.all(np.isfinite(W)):
        raise ValueError("non-finite weights are outside the quantizer's contract")
    lead = W.shape[:-1]
    blocks = W.reshape(-1, blocksize)

    # 1. absmax of each block (exact in fp32).
    absmax = np.max(np.abs(blocks), axis=1).astype(np.float32)

    # 2. normalise by IEEE fp32 division; zero blocks are handled below.
    safe = np.where(absmax == 0, np.float32(1), absmax).astype(np.float32)
    n = (blocks / safe[:, None]).astype(np.float32)

    # 3. code = number of midpoints strictly below n (nearest, ties -> lower).
    M = nf4_midpoints()
    codes = np.zeros(n.shape, dtype=np.uint8)
    for i in range(15):
        codes += (n > M[i]).astype(np.uint8)
    codes[absmax == 0, :] = 7

    # 4. pack: even element in the high nibble, odd element in the low one.
    codes = codes.reshape(*lead, K)
    packed = ((codes[..., 0::2] << 4) | codes[..., 1::2]).astype(np.uint8)
    return packed, absmax.reshape(*lead, K // blocksize)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """``packed uint8[..., K/2]`` -> ``codes uint8[..., K]``."""
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = packed >> 4
    out[..., 1::2] = packed & 0x0F
    return out


def dequantize_blockwise(packed: np.ndarray, absmax: np.ndarray,
                         blocksize: int = BLOCKSIZE) -> np.ndarray:
    """NF4 -> weights, ``w = L[code] * absmax`` evaluated exactly (fp64).

    ``packed[..., K/2]``, ``absmax[..., K/blocksize]`` -> ``float64[..., K]``.
    """
    codes = unpack_codes(packed)
    K = codes.shape[-1]
    L = nf4_levels().astype(np.float64)
    a = np.asarray(absmax, dtype=np.float32).astype(np.float64)
    a = a.reshape(codes.shape[:-1] + (K // blocksize,))
    w = L[codes].reshape(codes.shape[:-1] + (K // blocksize, blocksize))
    return (w * a[..., None]).reshape(codes.shape)
