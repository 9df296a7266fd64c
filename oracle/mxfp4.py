"""MXFP4 (e2m1 elements, e8m0 scale per 32) quantize / dequantize, from the format's definition.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What the pages fix: the kernel also serves MXFP4, the second sixteen-entry
codebook, computing on a checkpoint's exact released bytes ("grouped-nf4-gemm
& experts-4bit", jordananderson-pages.pages.dev, third bullet), and they name
its parts: e2m1 elements and e8m0 scales ("MoE Training on Consumer GPUs",
cerinamroth.com/ml, section "Task guides").  The format itself is the OCP
Microscaling (MX) specification v1.0; the readings taken here:

* element: FP4 E2M1 -- sign bit, 2 exponent bits (bias 1), 1 mantissa bit,
  exponent 0 subnormal, no infinities or NaN; magnitudes
  {0, 0.5, 1, 1.5, 2, 3, 4, 6}; code c in 0..15, bit 3 the sign;
* scale: E8M0 -- an unsigned 8-bit biased exponent, value 2^(b - 127); 255
  is NaN (never written here);
* block: 32 consecutive elements of a row along K (the reduction dimension)
  share one scale; ``w = 2^(b - 127) * e2m1(c)``;
* quantization (the specification's conversion rule): shared exponent
  ``floor(log2(max |x|)) - 2`` (2 = the largest E2M1 exponent), clamped to
  [-127, 127]; each ``x / 2^shared`` is rounded to the nearest E2M1 value, ties
  to even mantissa, magnitudes above 6 saturating to 6; an all-zero block gets
  b = 0 and codes 0;
* packing: two codes per byte with element 2j in the LOW nibble of byte j (the
  convention of released MXFP4 checkpoints; NF4's bitsandbytes layout is the
  other way round), ``packed uint8[..., N, K/2]``, ``scales uint8[..., N, K/32]``.
"""

from __future__ import annotations

import numpy as np

BLOCK = 32
E2M1_MAX = 6.0


def e2m1_values() -> np.ndarray:
    """The sixteen E2M1 values by code, fp64 (code 8 is -0)."""
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    return np.concatenate([mags, -mags])


def _round_e2m1(y: np.ndarray) -> np.ndarray:
    """Codes of the E2M1 values nearest to ``y`` (fp32), ties to even mantissa,
    saturating at +-6."""
    y = np.asarray(y, dtype=np.float32)
    mags = e2m1_values()[:8].astype(np.float32)
    a = np.minimum(np.abs(y), np.float32(E2M1_MAX))
    # distance to each magnitude; ties resolved toward the code with an even
    # mantissa bit (codes 0, 2, 4, 6 -- mantissa is the code's low bit)
    d = np.abs(a[..., None] - mags)
    best = np.argmin(d, axis=-1)
    dmin = np.take_along_axis(d, best[..., None], axis=-1)[..., 0]
    tie = np.sum(d == dmin[..., None], axis=-1) > 1
    # at a tie the two candidates are best and best + 1; take the even one
    best = np.where(tie & (best % 2 == 1), best + 1, best)
    sign = (np.signbit(y) & (best > 0)).astype(np.int64)
    return (best + 8 * sign).astype(np.uint8)


def quantize_mxfp4(W: np.ndarray):
    """``W float32[..., N, K]`` (K % 32 == 0) -> ``(packed uint8[..., N, K/2],
    scales uint8[..., N, K/32])``."""
    W = np.asarray(W, dtype=np.float32)
    K = W.shape[-1]
    if K % BLOCK:
        raise ValueError("K must be a multiple of 32")
    if not np.all(np.isfinite(W)):
        raise ValueError("non-finite weights are outside the quantizer's contract")
    g = W.reshape(W.shape[:-1] + (K // BLOCK, BLOCK))
    amax = np.abs(g).max(axis=-1)
    zero = amax == 0
    safe = np.where(zero, np.float32(1), amax)
    # floor(log2 amax) exactly: the unbiased exponent of the fp32 value
    # (frexp gives amax = m 2^ex with m in [0.5, 1))
    _, ex = np.frexp(safe.astype(np.float64))
    shared = np.clip(ex.astype(np.int64) - 1 - 2, -127, 127)
    y = (g.astype(np.float64) / np.exp2(shared.astype(np.float64))[..., None]).astype(np.float32)
    codes = _round_e2m1(y)
    codes = np.where(zero[..., None], 0, codes).astype(np.uint8)
    b = np.where(zero, 0, shared + 127).astype(np.uint8)
    c = codes.reshape(W.shape)
    packed = (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)
    return packed, b


def dequantize_mxfp4(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """``(packed uint8[..., N, K/2], scales uint8[..., N, K/32])`` -> fp64
    ``[..., N, K]``: ``2^(b - 127) * e2m1(code)``, exact."""
    packed = np.asarray(packed, dtype=np.uint8)
    scales = np.asarray(scales, dtype=np.uint8)
    if np.any(scales == 255):
        raise ValueError("scale byte 255 is NaN in E8M0")
    codes = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.int64)
    codes[..., 0::2] = packed & 0x0F
    codes[..., 1::2] = packed >> 4
    vals = e2m1_values()[codes]
    K = codes.shape[-1]
    v = vals.reshape(codes.shape[:-1] + (K // BLOCK, BLOCK))
    s = np.exp2(scales.astype(np.float64) - 127.0)
    return (v * s[..., None]).reshape(codes.shape)
