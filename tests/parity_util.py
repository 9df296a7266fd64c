"""Shared helpers of the GPU parity tests: tolerance metric and setups."""

from __future__ import annotations

import numpy as np
import torch

import moe_synth
import oracle

# Tolerance of the layer's floating-point outputs against the oracle:
#   rel_max = max_i |y_i - r_i| / max(|r_i|, RMS(r))  <= 1e-2
#   mae     = mean_i |y_i - r_i|                       <= 1e-3 * RMS(r)
REL_MAX = 1e-2
MAE_RMS = 1e-3


def errors(y, ref):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert y.shape == ref.shape and ref.size > 0
    rms = float(np.sqrt(np.mean(ref ** 2)))
    assert rms > 0, "reference is all zero: the comparison would be vacuous"
    rel = float(np.max(np.abs(y - ref) / np.maximum(np.abs(ref), rms)))
    mae = float(np.mean(np.abs(y - ref)))
    return rel, mae / rms


def assert_close_16bit(y, ref, dtype, what=""):
    """A 16-bit output against the oracle, both ways.

    Against the oracle value rounded once to ``dtype`` it must meet the full
    bar: that isolates the kernel's arithmetic from the final rounding.
    Against the unrounded oracle (the output's own rounding counted as error)
    it must meet rel_max <= 1e-2, and mae <= 1e-3 * RMS for fp16; for bf16 the
    rounding alone costs about 1e-3 * RMS on average (2^-9 of each value's
    power of two), so there the bound is 1e-3 * RMS plus the mean error of
    rounding the oracle itself to bf16."""
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    ref_rounded = torch.from_numpy(ref).to(dtype).double().numpy()
    r2 = assert_close(y, ref_rounded, f"{what} (oracle rounded to {dtype})")
    rel, mae = errors(y, ref)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    allowance = 0.0 if dtype == torch.float16 else float(np.mean(np.abs(ref_rounded - ref))) / rms
    assert rel <= REL_MAX and mae <= MAE_RMS + allowance, (
        f"{what} (unrounded oracle): rel_max={rel:.3e} mae/rms={mae:.3e} "
        f"(bound {MAE_RMS + allowance:.3e})")
    return (rel, mae), r2


def assert_close(y, ref, what=""):
    y = np.asarray(y, dtype=np.float64)
    assert np.all(np.isfinite(y)), f"{what}: non-finite GPU output"
    assert np.any(y != 0), f"{what}: GPU output is all zero"
    rel, mae = errors(y, ref)
    assert rel <= REL_MAX and mae <= MAE_RMS, f"{what}: rel_max={rel:.3e} mae/rms={mae:.3e}"
    return rel, mae


_STACKS = {}


def gpu_stack(shape, seed, device="cuda"):
    """Quantize the seeded fp32 stacks on the GPU (cached per shape and seed).

    Returns ``((packed_gu, absmax_gu, packed_d, absmax_d), (w_gu, w_d))`` with
    the fp32 weights kept on the device for the oracle to copy per expert."""
    import bit_mixture_experts_route_b200 as moe
    # the weights depend on these fields only, so shapes that differ in their
    # routing alone (uniform / Zipf) share one stack and its oracle experts
    key = (shape.E, shape.H, shape.I, shape.sigma, shape.outlier_frac, seed)
    if key not in _STACKS:
        _STACKS.clear()
        w_gu = moe_synth.weights(shape, "gate_up", seed, device=device)
        w_d = moe_synth.weights(shape, "down", seed, device=device)
        p_gu, a_gu = moe.nf4_quantize(w_gu)
        p_d, a_d = moe.nf4_quantize(w_d)
        _STACKS[key] = ((p_gu, a_gu, p_d, a_d), (w_gu, w_d))
    return _STACKS[key]


class LazyOracleStack:
    """The oracle's expert stack, quantized one expert at a time from the
    fp32 weights, each expert's codes and absmax checked bit-exact against the
    GPU's on first use.  Same interface as ``oracle.ExpertStack``."""

    _shared = {}

    @classmethod
    def shared(cls, stack_gpu, weights_fp32):
        """One instance per GPU stack, so tests on the same weights reuse the
        experts already quantized and checked."""
        key = id(stack_gpu[0])
        if key not in cls._shared:
            cls._shared.clear()
            cls._shared[key] = cls(stack_gpu, weights_fp32)
        return cls._shared[key]

    def __init__(self, stack_gpu, weights_fp32):
        self.gpu = stack_gpu
        self.w_gu, self.w_d = weights_fp32
        self.E, two_i, self.H = self.w_gu.shape
        self.I = two_i // 2
        self._gu, self._d = {}, {}
        self.checked = 0

    def _quant(self, w_dev, packed_dev, absmax_dev, e):
        w = w_dev[e].cpu().numpy()
        p, a = oracle.quantize_blockwise(w)
        assert np.array_equal(packed_dev[e].cpu().numpy(), p), f"codes differ, expert {e}"
        assert np.array_equal(absmax_dev[e].cpu().numpy().view(np.int32),
                              a.reshape(-1).view(np.int32)), f"absmax differs, expert {e}"
        self.checked += 1
        return oracle.dequantize_blockwise(p, a)

    def gate_up(self, e):
        if e not in self._gu:
            self._gu[e] = self._quant(self.w_gu, self.gpu[0], self.gpu[1], e)
        return self._gu[e]

    def down(self, e):
        if e not in self._d:
            self._d[e] = self._quant(self.w_d, self.gpu[2], self.gpu[3], e)
        return self._d[e]


def run_layer_steps(X, logits, k, renorm, stack_gpu, algo="auto", h_dtype=torch.float16,
                    yp_dtype=torch.float16):
    """The layer through the five exported calls, one by one."""
    import bit_mixture_experts_route_b200 as moe
    p_gu, a_gu, p_d, a_d = stack_gpu
    T = X.shape[0]
    r = moe.route_permute(logits, k, renorm)
    M = T * k
    Hh = moe.nf4_grouped_gemm(X, p_gu, a_gu, r["expert_offsets"], M, gather=r["sorted_rows"],
                              k=k, epilogue="swiglu", out_dtype=h_dtype, algo=algo)
    Yp = moe.nf4_grouped_gemm(Hh, p_d, a_d, r["expert_offsets"], M, epilogue="none",
                              out_dtype=yp_dtype, algo=algo)
    Y = moe.unpermute_combine(Yp, r["inv_perm"], r["topk_w"])
    return Y, r, Hh, Yp
