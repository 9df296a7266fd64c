"""The C-ABI library loads and exports what include/moe_nf4.h declares (CPU).

No compute call is made: the host-only entry points (status strings, levels,
workspace sizes) are exercised, and argument validation is checked on calls
that must be rejected before any CUDA call.
"""

import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from bit_mixture_experts_route_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_nf4.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from bit_mixture_experts_route_b200 import build
        build.build()
    return _lib.load()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_five_path_calls():
    names = _declared()
    for n in ("moe_nf4_quantize", "moe_route_permute", "moe_nf4_grouped_gemm", "moe_swiglu",
              "moe_unpermute_combine"):
        assert n in names


def test_every_declared_symbol_is_exported_and_bound(lib):
    for name in _declared():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def test_abi_version_and_status_strings(lib):
    assert lib.moe_abi_version() == 3
    for code, name in _lib.STATUS.items():
        assert lib.moe_status_string(code).decode() == name


def test_library_levels_equal_oracle_levels_bitwise(lib):
    got = np.array(_lib.nf4_levels(), dtype=np.float32)
    assert np.array_equal(got.view(np.int32), oracle.nf4_levels().view(np.int32))


def test_route_workspace_size(lib):
    n = _lib.route_permute_workspace_size(4096, 128, 8)
    assert n >= 4096 * 8 * 4 + 64 * 128 * 4
    with pytest.raises(_lib.MoEError):
        _lib.route_permute_workspace_size(16, 8, 9)   # k > E
    with pytest.raises(_lib.MoEError):
        _lib.route_permute_workspace_size(16, 2048, 8)  # E > 1024


def test_layer_workspace_size(lib):
    n = _lib.layer_workspace_size(64, 64, 8, 2048, 1024)
    assert n >= 64 * 8 * (1024 + 2048) * 2


# Fake, never-dereferenced device addresses: validation must reject these
# calls before touching CUDA.
ALIGNED = ctypes.c_void_p(0x7000_0000)
MISALIGNED = ctypes.c_void_p(0x7000_0004)


def test_quantize_rejects_bad_arguments(lib):
    q = lib.moe_nf4_quantize
    assert q(ALIGNED, 1, 64, 100, 64, ALIGNED, ALIGNED, None, None) == 1   # K % 64
    assert q(ALIGNED, 1, 64, 128, 32, ALIGNED, ALIGNED, None, None) == 1   # blocksize
    assert q(None, 1, 64, 128, 64, ALIGNED, ALIGNED, None, None) == 1      # null W
    assert q(MISALIGNED, 1, 64, 128, 64, ALIGNED, ALIGNED, None, None) == 2


def test_grouped_gemm_rejects_bad_arguments(lib):
    g = lib.moe_nf4_grouped_gemm
    args = dict(A=ALIGNED, adt=1, arows=32, gather=ALIGNED, k=8, packed=ALIGNED, absmax=ALIGNED,
                off=ALIGNED, E=8, N=1024, K=256, M=32, epi=1, out=ALIGNED, odt=0, algo=0,
                err=None, s=None)

    def call(**kw):
        a = dict(args, **kw)
        return g(*a.values())

    assert call(adt=0) == 1            # fp32 activations are not accepted
    assert call(K=100) == 1            # K % 64
    assert call(N=100) == 1            # N % 64
    assert call(epi=7) == 1
    assert call(algo=9) == 1
    assert call(E=0) == 1
    assert call(packed=None) == 1
    assert call(out=MISALIGNED) == 2
    assert call(gather=None, arows=10) == 1   # without gather A needs M_total rows


def test_route_permute_rejects_small_workspace(lib):
    r = lib.moe_route_permute
    assert r(ALIGNED, 16, 8, 2, 1, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 8,
             None) == 4
    assert r(ALIGNED, 16, 8, 9, 1, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED,
             1 << 20, None) == 1


def test_binding_fails_loudly_without_the_library(monkeypatch):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", "/nonexistent/libmoenf4.so")
    with pytest.raises(_lib.MoEError):
        _lib.load()


def test_int4_calls_reject_bad_arguments(lib):
    A, M = ALIGNED, MISALIGNED
    # quantize: K % 128, null, misaligned
    assert lib.moe_int4_quantize(A, 1, 8, 192, A, A, None, None) == 1
    assert lib.moe_int4_quantize(None, 1, 8, 256, A, A, None, None) == 1
    assert lib.moe_int4_quantize(A, 1, 8, 256, M, A, None, None) == 2
    # grouped GEMM: N % 128 or K % 256 -> unsupported; bad epilogue / dtype;
    # A_rows < M_total; misaligned output
    # (..., epilogue, out, out_dtype, algo, dev_err, stream); K = 384 has no
    # GEMV form (K % 256) but a tensor-core one (K % 128)
    g4 = lib.moe_int4_grouped_gemm
    assert g4(A, 8, A, A, A, 2, 64, 256, 8, 0, A, 0, 0, None, None) == 3
    assert g4(A, 8, A, A, A, 2, 128, 384, 8, 0, A, 0, 1, None, None) == 3
    assert g4(A, 8, A, A, A, 2, 128, 192, 8, 0, A, 0, 2, None, None) == 3
    assert g4(A, 8, A, A, A, 2, 128, 256, 8, 7, A, 0, 0, None, None) == 1
    assert g4(A, 8, A, A, A, 2, 128, 256, 8, 0, A, 9, 0, None, None) == 1
    assert g4(A, 8, A, A, A, 2, 128, 256, 8, 0, A, 0, 5, None, None) == 1
    assert g4(A, 4, A, A, A, 2, 128, 256, 8, 0, A, 0, 0, None, None) == 1
    assert g4(A, 8, A, A, A, 2, 128, 256, 8, 0, M, 0, 0, None, None) == 2


def test_lora_delta_rejects_bad_arguments(lib):
    A, M = ALIGNED, MISALIGNED
    # (X, A_rows, offsets, E, N, K, r, lora_A, lora_B, scale, M_total, out, dev_err, stream)
    # rank outside 8..64 or not a multiple of 8, K % 8, E > 1024 -> unsupported
    assert lib.moe_lora_delta(A, 8, A, 2, 64, 256, 4, A, A, 1.0, 8, A, None, None) == 3
    assert lib.moe_lora_delta(A, 8, A, 2, 64, 256, 12, A, A, 1.0, 8, A, None, None) == 3
    assert lib.moe_lora_delta(A, 8, A, 2, 64, 256, 72, A, A, 1.0, 8, A, None, None) == 3
    assert lib.moe_lora_delta(A, 8, A, 2, 64, 260, 16, A, A, 1.0, 8, A, None, None) == 3
    assert lib.moe_lora_delta(A, 8, A, 1025, 64, 256, 16, A, A, 1.0, 8, A, None, None) == 3
    # A_rows < M_total, null adapters, misaligned output
    assert lib.moe_lora_delta(A, 4, A, 2, 64, 256, 16, A, A, 1.0, 8, A, None, None) == 1
    assert lib.moe_lora_delta(A, 8, A, 2, 64, 256, 16, None, A, 1.0, 8, A, None, None) == 1
    assert lib.moe_lora_delta(A, 8, A, 2, 64, 256, 16, A, A, 1.0, 8, M, None, None) == 2


def test_mxfp4_calls_reject_bad_arguments(lib):
    A, M = ALIGNED, MISALIGNED
    # quantize: K % 32, null, misaligned
    assert lib.moe_mxfp4_quantize(A, 1, 8, 48, A, A, None, None) == 1
    assert lib.moe_mxfp4_quantize(A, 1, 8, 64, A, None, None, None) == 1
    assert lib.moe_mxfp4_quantize(A, 1, 8, 64, A, M, None, None) == 2
    # grouped GEMM (..., epilogue, out, out_dtype, algo, dev_err, stream):
    # N % 128 or K % 64 -> unsupported by both kernels; K % 256 != 0 ->
    # unsupported by the GEMV; bad epilogue / dtype / algo; A_rows < M_total;
    # misaligned scales
    g = lib.moe_mxfp4_grouped_gemm
    assert g(A, 8, A, A, A, 2, 64, 256, 8, 0, A, 0, 0, None, None) == 3
    assert g(A, 8, A, A, A, 2, 128, 288, 8, 0, A, 0, 0, None, None) == 3
    assert g(A, 8, A, A, A, 2, 128, 320, 8, 0, A, 0, 1, None, None) == 3
    assert g(A, 8, A, A, A, 2, 64, 320, 8, 0, A, 0, 2, None, None) == 3
    assert g(A, 8, A, A, A, 2, 128, 256, 8, 5, A, 0, 0, None, None) == 1
    assert g(A, 8, A, A, A, 2, 128, 256, 8, 0, A, 4, 0, None, None) == 1
    assert g(A, 8, A, A, A, 2, 128, 256, 8, 0, A, 0, 7, None, None) == 1
    assert g(A, 4, A, A, A, 2, 128, 256, 8, 0, A, 0, 0, None, None) == 1
    assert g(A, 8, A, M, A, 2, 128, 256, 8, 0, A, 0, 0, None, None) == 2


def test_backward_calls_reject_bad_arguments(lib):
    A, M = ALIGNED, MISALIGNED
    # transposed GEMM: (G, g_dtype, G_rows, packed, absmax, offsets, E, N, K, M_total, out,
    # out_dtype, algo, dev_err, stream): bf16 G, K % 64, G_rows < M_total, misaligned out,
    # bad algo; the tensor-core form needs fp16 G and K % 256
    t = lib.moe_nf4_grouped_gemm_t
    assert t(A, 1, 8, A, A, A, 2, 128, 256, 8, A, 0, 0, None, None) == 1
    assert t(A, 0, 8, A, A, A, 2, 128, 96, 8, A, 0, 0, None, None) == 1
    assert t(A, 0, 4, A, A, A, 2, 128, 256, 8, A, 0, 0, None, None) == 1
    assert t(A, 0, 8, A, A, A, 2, 128, 256, 8, M, 0, 0, None, None) == 2
    assert t(A, 0, 8, A, A, A, 2, 128, 256, 8, A, 0, 9, None, None) == 1
    assert t(A, 0, 8, A, A, A, 2, 128, 256, 8, A, 0, 2, None, None) == 3
    assert t(A, 2, 8, A, A, A, 2, 128, 192, 8, A, 0, 2, None, None) == 3
    # fused down backward (dYp, G_rows, packed, absmax, offsets, E, H, I, M_total, gu, dgu,
    # dgu_dtype, dev_err, stream): I % 256, bf16 output, null gu
    d = lib.moe_nf4_down_backward
    assert d(A, 8, A, A, A, 2, 128, 192, 8, A, A, 0, None, None) == 3
    assert d(A, 8, A, A, A, 2, 128, 256, 8, A, A, 1, None, None) == 1
    assert d(A, 8, A, A, A, 2, 128, 256, 8, None, A, 0, None, None) == 1
    # SwiGLU backward: bf16 inputs, null dh
    assert lib.moe_swiglu_backward(A, A, 1, 4, 8, A, 0, None) == 1
    assert lib.moe_swiglu_backward(A, None, 0, 4, 8, A, 0, None) == 1
    # combine backward: k > 32, misaligned dw
    assert lib.moe_combine_backward(A, A, 0, A, A, 2, 33, 8, A, 0, A, None, None) == 1
    assert lib.moe_combine_backward(A, A, 0, A, A, 2, 2, 8, A, 0, M, None, None) == 2
    # routing backward: k > E, E > 1024
    assert lib.moe_route_backward(A, A, A, A, 2, 4, 5, 1, A, None, None) == 1
    assert lib.moe_route_backward(A, A, A, A, 2, 2048, 8, 1, A, None, None) == 1
