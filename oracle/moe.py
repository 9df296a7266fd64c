"""The NF4 mixture-of-experts layer, per token and per expert, in fp64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The layer the library computes ("grouped-nf4-gemm & experts-4bit",
jordananderson-pages.pages.dev, first bullet: MoE matmuls run directly on the
NF4 weights; the problem statement: gate_up, SiLU(gate)*up, down, a
routing-weighted combine).  Readings taken where the pages are silent:

* the fused stacks are ``W_gu[E, 2I, H]`` and ``W_d[E, H, I]`` (out x in per
  expert); rows [0, I) of ``W_gu[e]`` are the gate, rows [I, 2I) the up
  projection (concatenated, not interleaved);
* silu(g) = g / (1 + exp(-g));
* the output is y_t = sum_j w[t, j] * W_d[e_j] (silu(g_j) * u_j), summed in
  j order.

The oracle evaluates this on the dequantized weights (exact fp64 products
of the fp32 level and fp32 absmax), so quantization error is part of the
definition, not of the GPU's error.  Activations enter as the exact values
of their bf16 inputs; all arithmetic is fp64.
"""

from __future__ import annotations

import numpy as np

from .int4 import dequantize_int4_grouped
from .mxfp4 import dequantize_mxfp4
from .nf4 import dequantize_blockwise
from .routing import route_topk, permute_by_expert


class ExpertStack:
    """NF4 gate_up and down stacks of one layer, dequantized lazily per expert.

    ``packed_gu uint8[E, 2I, H/2]``, ``absmax_gu float32[E, 2I*H/64]``,
    ``packed_d uint8[E, H, I/2]``, ``absmax_d float32[E, H*I/64]``.
    """

    def __init__(self, packed_gu, absmax_gu, packed_d, absmax_d):
        self.packed_gu = np.asarray(packed_gu, dtype=np.uint8)
        self.absmax_gu = np.asarray(absmax_gu, dtype=np.float32)
        self.packed_d = np.asarray(packed_d, dtype=np.uint8)
        self.absmax_d = np.asarray(absmax_d, dtype=np.float32)
        self.E, two_i, half_h = self.packed_gu.shape
        self.I = two_i // 2
        self.H = half_h * 2
        assert self.packed_d.shape == (self.E, self.H, self.I // 2)
        self._gu = {}
        self._d = {}

    def gate_up(self, e: int) -> np.ndarray:
        """fp64 ``[2I, H]``: rows [0, I) gate, [I, 2I) up."""
        if e not in self._gu:
            self._gu[e] = dequantize_blockwise(
                self.packed_gu[e], self.absmax_gu[e].reshape(2 * self.I, -1))
        return self._gu[e]

    def down(self, e: int) -> np.ndarray:
        """fp64 ``[H, I]``."""
        if e not in self._d:
            self._d[e] = dequantize_blockwise(
                self.packed_d[e], self.absmax_d[e].reshape(self.H, -1))
        return self._d[e]


class Int4ExpertStack:
    """Grouped INT4 gate_up and down stacks of one layer (``oracle.int4``),
    dequantized lazily per expert; same interface as ``ExpertStack``.

    ``packed_gu uint8[E, 2I, H/2]``, ``meta_gu uint32[E, 2I, H/128]``,
    ``packed_d uint8[E, H, I/2]``, ``meta_d uint32[E, H, I/128]``.
    """

    def __init__(self, packed_gu, meta_gu, packed_d, meta_d):
        self.packed_gu, self.meta_gu = np.asarray(packed_gu, np.uint8), np.asarray(meta_gu)
        self.packed_d, self.meta_d = np.asarray(packed_d, np.uint8), np.asarray(meta_d)
        self.E, two_i, half_h = self.packed_gu.shape
        self.I = two_i // 2
        self.H = half_h * 2
        assert self.packed_d.shape == (self.E, self.H, self.I // 2)
        self._gu, self._d = {}, {}

    def gate_up(self, e: int) -> np.ndarray:
        if e not in self._gu:
            self._gu[e] = dequantize_int4_grouped(self.packed_gu[e], self.meta_gu[e])
        return self._gu[e]

    def down(self, e: int) -> np.ndarray:
        if e not in self._d:
            self._d[e] = dequantize_int4_grouped(self.packed_d[e], self.meta_d[e])
        return self._d[e]


class Mxfp4ExpertStack:
    """MXFP4 gate_up and down stacks of one layer (``oracle.mxfp4``),
    dequantized lazily per expert; same interface as ``ExpertStack``.

    ``packed_gu uint8[E, 2I, H/2]``, ``scales_gu uint8[E, 2I, H/32]``,
    ``packed_d uint8[E, H, I/2]``, ``scales_d uint8[E, H, I/32]``.
    """

    def __init__(self, packed_gu, scales_gu, packed_d, scales_d):
        self.packed_gu, self.scales_gu = np.asarray(packed_gu, np.uint8), np.asarray(scales_gu)
        self.packed_d, self.scales_d = np.asarray(packed_d, np.uint8), np.asarray(scales_d)
        self.E, two_i, half_h = self.packed_gu.shape
        self.I = two_i // 2
        self.H = half_h * 2
        assert self.packed_d.shape == (self.E, self.H, self.I // 2)
        self._gu, self._d = {}, {}

    def gate_up(self, e: int) -> np.ndarray:
        if e not in self._gu:
            self._gu[e] = dequantize_mxfp4(self.packed_gu[e], self.scales_gu[e])
        return self._gu[e]

    def down(self, e: int) -> np.ndarray:
        if e not in self._d:
            self._d[e] = dequantize_mxfp4(self.packed_d[e], self.scales_d[e])
        return self._d[e]


def _silu(g: np.ndarray) -> np.ndarray:
    return g / (1.0 + np.exp(-g))


def swiglu(gu: np.ndarray) -> np.ndarray:
    """``gu[M, 2I]`` -> ``h[M, I] = silu(gu[:, :I]) * gu[:, I:]`` in fp64."""
    gu = np.asarray(gu, dtype=np.float64)
    I = gu.shape[1] // 2
    return _silu(gu[:, :I]) * gu[:, I:]


def _grouped(A, weight_of, N: int, expert_offsets, gather, k: int, rows) -> np.ndarray:
    """``out[p] = W(e(p)) @ A[r(p)]`` for the positions p of a grouped GEMM;
    ``weight_of(e)`` returns expert e's dequantized ``[N, K]`` weights."""
    A = np.asarray(A, dtype=np.float64)
    offsets = np.asarray(expert_offsets, dtype=np.int64)
    M_total = int(offsets[-1])
    positions = np.arange(M_total) if rows is None else np.asarray(rows)
    out = np.zeros((positions.size, N), dtype=np.float64)
    experts = np.searchsorted(offsets, positions, side="right") - 1
    cache = {}
    for i, p in enumerate(positions):
        e = int(experts[i])
        if e not in cache:
            cache[e] = weight_of(e)
        r = int(gather[p]) // k if gather is not None else int(p)
        out[i] = cache[e] @ A[r]
    return out


def grouped_gemm(A: np.ndarray, packed: np.ndarray, absmax: np.ndarray,
                 expert_offsets: np.ndarray, gather=None, k: int = 1,
                 rows=None) -> np.ndarray:
    """One grouped NF4 GEMM: ``out[p] = W[e(p)] @ A[r(p)]``.

    ``packed uint8[E, N, K/2]``, ``absmax float32[E, N*K/64]``; e(p) is the
    expert whose segment [offsets[e], offsets[e+1]) holds position p; r(p) is
    ``gather[p] // k`` when a gather list (``sorted_rows``) is given, else p.
    ``rows`` optionally restricts the result to those positions (returned in
    that order).  fp64 result ``[len(rows) or M_total, N]``.
    """
    E, N, half_k = packed.shape
    return _grouped(A, lambda e: dequantize_blockwise(packed[e], absmax[e].reshape(N, -1)), N,
                    expert_offsets, gather, k, rows)


def grouped_gemm_int4(A: np.ndarray, packed: np.ndarray, meta: np.ndarray,
                      expert_offsets: np.ndarray, gather=None, k: int = 1,
                      rows=None) -> np.ndarray:
    """The same grouped GEMM on grouped INT4 weights (``oracle.int4``):
    ``packed uint8[E, N, K/2]``, ``meta uint32[E, N, K/128]``."""
    E, N, half_k = packed.shape
    return _grouped(A, lambda e: dequantize_int4_grouped(packed[e], meta[e]), N, expert_offsets,
                    gather, k, rows)


def grouped_gemm_mxfp4(A: np.ndarray, packed: np.ndarray, scales: np.ndarray,
                       expert_offsets: np.ndarray, gather=None, k: int = 1,
                       rows=None) -> np.ndarray:
    """The same grouped GEMM on MXFP4 weights (``oracle.mxfp4``):
    ``packed uint8[E, N, K/2]``, ``scales uint8[E, N, K/32]``."""
    E, N, half_k = packed.shape
    return _grouped(A, lambda e: dequantize_mxfp4(packed[e], scales[e]), N, expert_offsets,
                    gather, k, rows)


def unpermute_combine(Yp: np.ndarray, inv_perm: np.ndarray,
                      weights: np.ndarray) -> np.ndarray:
    """``Y[t] = sum_j weights[t, j] * Yp[inv_perm[t*k + j]]`` (j order), fp64."""
    Yp = np.asarray(Yp, dtype=np.float64)
    weights = np.asarray(weights, dtype=np.float64)
    T, k = weights.shape
    Y = np.zeros((T, Yp.shape[1]), dtype=np.float64)
    for t in range(T):
        for j in range(k):
            Y[t] += weights[t, j] * Yp[int(inv_perm[t * k + j])]
    return Y


def moe_layer(x: np.ndarray, logits: np.ndarray, stack: ExpertStack, k: int,
              renormalize: bool = True, tokens=None) -> np.ndarray:
    """The layer, one token and one routed expert at a time.

    ``x[T, H]`` holds the activations' exact values (bf16 inputs widened);
    ``logits float32[T, E]``.  Returns fp64 ``Y[len(tokens) or T, H]``.
    """
    x = np.asarray(x, dtype=np.float64)
    idx, w = route_topk(np.asarray(logits, dtype=np.float32), k, renormalize)
    toks = range(x.shape[0]) if tokens is None else tokens
    I = stack.I
    out = []
    for t in toks:
        y = np.zeros(stack.H, dtype=np.float64)
        for j in range(k):
            e = int(idx[t, j])
            gu = stack.gate_up(e) @ x[t]
            h = _silu(gu[:I]) * gu[I:]
            y += w[t, j] * (stack.down(e) @ h)
        out.append(y)
    return np.stack(out) if out else np.zeros((0, stack.H))


def moe_layer_dense(x: np.ndarray, logits: np.ndarray, stack: ExpertStack,
                    k: int, renormalize: bool = True) -> np.ndarray:
    """Brute force: every expert on every token, weighted by a dense gate.

    ``Y = sum_e G[:, e] * MLP_e(X)`` with ``G[T, E]`` zero off the top-k.  A
    second formulation of ``moe_layer`` (batched over tokens, no permutation)
    used to pin it.
    """
    x = np.asarray(x, dtype=np.float64)
    idx, w = route_topk(np.asarray(logits, dtype=np.float32), k, renormalize)
    T = x.shape[0]
    G = np.zeros((T, stack.E), dtype=np.float64)
    np.put_along_axis(G, idx.astype(np.int64), w, axis=1)
    I = stack.I
    Y = np.zeros((T, stack.H), dtype=np.float64)
    for e in range(stack.E):
        GU = x @ stack.gate_up(e).T
        Hh = _silu(GU[:, :I]) * GU[:, I:]
        Y += G[:, e:e + 1] * (Hh @ stack.down(e).T)
    return Y


def moe_layer_permuted(x, logits, stack: ExpertStack, k: int,
                       renormalize: bool = True) -> np.ndarray:
    """The same layer through the explicit route -> permute -> grouped gate_up
    -> SwiGLU -> grouped down -> combine steps, as the library runs them."""
    x = np.asarray(x, dtype=np.float64)
    idx, w = route_topk(np.asarray(logits, dtype=np.float32), k, renormalize)
    offsets, sorted_rows, inv_perm = permute_by_expert(idx, stack.E)
    GU = grouped_gemm(x, stack.packed_gu, stack.absmax_gu, offsets,
                      gather=sorted_rows, k=k)
    Hh = swiglu(GU)
    Yp = grouped_gemm(Hh, stack.packed_d, stack.absmax_d, offsets)
    return unpermute_combine(Yp, inv_perm, w)
