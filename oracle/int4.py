"""Grouped asymmetric INT4 quantize / dequantize, written out from its definition.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What the pages fix: the experts can also be served as GPTQ-calibrated int4
weights through a single-token INT4 decode GEMV over the routed experts
("Jordan Anderson", jordananderson-pages.pages.dev, section
"grouped-nf4-gemm & experts-4bit", third bullet; "MoE Training on Consumer
GPUs", cerinamroth.com/ml, section "Task guides").  They print no packing,
group size or rounding rule.  The readings taken here follow the GPTQ
checkpoint convention:

* codes: unsigned 4-bit q in 0..15, asymmetric, one fp16 scale s and one
  4-bit zero z per group of 128 consecutive elements of a row (the input
  dimension K, the reduction dimension); ``w = (q - z) * s``;
* the group's range always contains 0: lo = min(min x, 0), hi = max(max x, 0);
* s = fp16(fl32((hi - lo) / 15)) (IEEE fp32 division, then round to nearest
  even fp16); every later step uses that stored fp16 value;
* z = clamp(rint(fl32(-lo / s)), 0, 15) and q = clamp(rint(fl32(x / s)) + z,
  0, 15), with rint rounding half to even (round to nearest);
* a group whose stored scale is 0 (all zeros) gets z = 0 and every q = 0;
* GPTQ's data-driven calibration chooses different codes in the same format;
  without calibration data the codes here are round-to-nearest.  The GEMV
  consumes any codes, so parity does not depend on how they were chosen;
* packing: two codes per byte, element 2j of a row in the HIGH nibble of byte
  j (the NF4 path's order), ``packed uint8[..., N, K/2]``;
* meta: one uint32 per group, ``fp16 bits of s | z << 16``,
  ``meta uint32[..., N, K/128]``.
"""

from __future__ import annotations

import numpy as np

GROUP = 128


def quantize_int4_grouped(W: np.ndarray):
    """``W float32[..., N, K]`` (K % 128 == 0) -> ``(packed uint8[..., N, K/2],
    meta uint32[..., N, K/128])``."""
    W = np.asarray(W, dtype=np.float32)
    K = W.shape[-1]
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    g = W.reshape(W.shape[:-1] + (K // GROUP, GROUP))
    lo = np.minimum(g.min(axis=-1), np.float32(0))
    hi = np.maximum(g.max(axis=-1), np.float32(0))
    s32 = ((hi - lo) / np.float32(15)).astype(np.float32)
    s16 = s32.astype(np.float16)
    s = s16.astype(np.float32)
    zero = s == 0
    safe = np.where(zero, np.float32(1), s)
    z = np.clip(np.rint((-lo / safe).astype(np.float32)), 0, 15)
    z = np.where(zero, 0, z).astype(np.int32)
    q = np.rint((g / safe[..., None]).astype(np.float32)).astype(np.int32) + z[..., None]
    q = np.clip(q, 0, 15)
    q = np.where(zero[..., None], 0, q).astype(np.uint8)
    codes = q.reshape(W.shape)
    packed = ((codes[..., 0::2] << 4) | codes[..., 1::2]).astype(np.uint8)
    meta = s16.view(np.uint16).astype(np.uint32) | (z.astype(np.uint32) << 16)
    return packed, meta


def int4_scales_zeros(meta: np.ndarray):
    """``meta uint32[...]`` -> ``(s float32[...], z int32[...])``."""
    meta = np.asarray(meta, dtype=np.uint32)
    s = (meta & 0xFFFF).astype(np.uint16).view(np.float16).astype(np.float32)
    z = ((meta >> 16) & 0xF).astype(np.int32)
    return s, z


def dequantize_int4_grouped(packed: np.ndarray, meta: np.ndarray) -> np.ndarray:
    """``(packed uint8[..., N, K/2], meta uint32[..., N, K/128])`` ->
    ``float64[..., N, K]``: ``(q - z) * s``, exact in fp64."""
    packed = np.asarray(packed, dtype=np.uint8)
    codes = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.int32)
    codes[..., 0::2] = packed >> 4
    codes[..., 1::2] = packed & 0x0F
    s, z = int4_scales_zeros(meta)
    K = codes.shape[-1]
    c = codes.reshape(codes.shape[:-1] + (K // GROUP, GROUP))
    w = (c - z[..., None]).astype(np.float64) * s[..., None].astype(np.float64)
    return w.reshape(codes.shape)
