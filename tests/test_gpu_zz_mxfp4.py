"""GPU parity of the MXFP4 path (quantize bit-exact, decode GEMV within
tolerance) against the CPU oracle (``oracle.mxfp4``).

The MXFP4 quantize and decode GEMV were first checked on a B200 through the C ABI alone
(``tests/c_abi``); this file checks them through the Python binding.  The
file name sorts after the forward-path GPU tests.
"""

import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_close, assert_close_16bit

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("bit_mixture_experts_route_b200")


def _np(t):
    return t.detach().cpu().numpy()


@pytest.mark.parametrize("E,N,K,outliers", [(2, 128, 512, False), (3, 256, 768, True), (1, 5, 96, False)])
def test_mxfp4_quantize_bit_exact(E, N, K, outliers):
    g = torch.Generator().manual_seed(K + N)
    W = torch.randn((E, N, K), generator=g) * 0.02
    if outliers:
        W[torch.rand((E, N, K), generator=g) < 1e-3] *= 30.0
    W[0, 3, :32] = 0.0                                   # an all-zero block
    W[0, 1, 32:64] = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 4)  # midpoints
    W[0, 2, :32] = torch.randn(32, generator=g) * 2.0 ** -135                     # subnormals
    packed, scales = moe.mxfp4_quantize(W.cuda())
    torch.cuda.synchronize()
    p_ref, s_ref = oracle.quantize_mxfp4(W.numpy())
    assert np.array_equal(_np(packed), p_ref)
    assert np.array_equal(_np(scales), s_ref)


def test_mxfp4_quantize_flags_nonfinite():
    W = torch.zeros((1, 128, 256))
    W[0, 7, 9] = float("nan")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.mxfp4_quantize(W.cuda(), dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & moe.DEVERR_NONFINITE


def _ragged(counts):
    off = np.zeros(len(counts) + 1, dtype=np.int32)
    off[1:] = np.cumsum(counts)
    return off


@pytest.mark.parametrize("epi", ["none", "swiglu"])
@pytest.mark.parametrize("counts", [[1, 0, 9, 16, 17, 40], [8, 8, 0, 3]])
def test_mxfp4_grouped_gemm_ragged(epi, counts):
    E = len(counts)
    off = _ragged(counts)
    M = int(off[-1])
    g = torch.Generator().manual_seed(sum(counts) + len(epi))
    N, K = (256, 768) if epi == "swiglu" else (384, 512)
    W = torch.randn((E, N, K), generator=g) * 0.03
    X = torch.randn((M, K), generator=g).to(torch.float16)
    packed, scales = moe.mxfp4_quantize(W.cuda())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = moe.mxfp4_grouped_gemm(X.cuda(), packed, scales, torch.from_numpy(off).cuda(), M,
                                 epilogue=epi, out_dtype=torch.float32, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    p_ref, s_ref = oracle.quantize_mxfp4(W.numpy())
    ref = oracle.grouped_gemm_mxfp4(X.float().numpy(), p_ref, s_ref, off)
    if epi == "swiglu":
        ref = oracle.swiglu(ref)
    assert_close(_np(out), ref, f"mxfp4 {epi} {counts}")


@pytest.mark.parametrize("out_dtype", [torch.float16, torch.bfloat16])
def test_mxfp4_grouped_gemm_output_dtypes(out_dtype):
    E, N, K = 2, 128, 256
    off = _ragged([5, 12])
    M = int(off[-1])
    g = torch.Generator().manual_seed(7)
    W = torch.randn((E, N, K), generator=g) * 0.05
    X = torch.randn((M, K), generator=g).to(torch.float16)
    packed, scales = moe.mxfp4_quantize(W.cuda())
    out = moe.mxfp4_grouped_gemm(X.cuda(), packed, scales, torch.from_numpy(off).cuda(), M,
                                 out_dtype=out_dtype)
    torch.cuda.synchronize()
    p_ref, s_ref = oracle.quantize_mxfp4(W.numpy())
    ref = oracle.grouped_gemm_mxfp4(X.float().numpy(), p_ref, s_ref, off)
    assert_close_16bit(out.double().cpu().numpy(), ref, out_dtype, f"mxfp4 out {out_dtype}")


def test_mxfp4_scale_out_of_exact_range_is_flagged():
    E, N, K = 1, 128, 256
    off = _ragged([4])
    W = torch.randn((E, N, K)) * 0.05
    packed, scales = moe.mxfp4_quantize(W.cuda())
    scales[0, 0, 0] = 150                                 # 2^23: products overflow fp16
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.mxfp4_grouped_gemm(torch.zeros((4, K), dtype=torch.float16, device="cuda"), packed,
                           scales, torch.from_numpy(off).cuda(), 4, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & moe.DEVERR_RANGE


def test_mxfp4_bad_offsets_flagged():
    E, N, K = 2, 128, 256
    packed = torch.zeros((E, N, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.full((E, N, K // 32), 127, dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.mxfp4_grouped_gemm(torch.zeros((8, K), dtype=torch.float16, device="cuda"), packed, scales,
                           torch.tensor([0, 6, 4], dtype=torch.int32, device="cuda"), 8,
                           dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & moe.DEVERR_BAD_OFFSETS
