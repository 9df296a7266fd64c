"""GPU parity of the grouped INT4 path (quantize bit-exact, decode GEMV
within tolerance) against the CPU oracle (``oracle.int4``)."""

import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_close, assert_close_16bit

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("bit_mixture_experts_route_b200")


def _np(t):
    return t.detach().cpu().numpy()


@pytest.mark.parametrize("E,N,K,outliers", [(2, 128, 512, False), (3, 256, 768, True)])
def test_int4_quantize_bit_exact(E, N, K, outliers):
    g = torch.Generator().manual_seed(K)
    W = torch.randn((E, N, K), generator=g) * 0.02
    if outliers:
        mask = torch.rand((E, N, K), generator=g) < 1e-3
        W[mask] *= 8.0
    W[0, 3, :128] = 0.0                     # an all-zero group
    W[1, 5, 128:256] = 0.37                 # a constant group
    packed, meta = moe.int4_quantize(W.cuda())
    torch.cuda.synchronize()
    p_ref, m_ref = oracle.quantize_int4_grouped(W.numpy())
    assert np.array_equal(_np(packed), p_ref)
    assert np.array_equal(_np(meta).view(np.uint32), m_ref)


def test_int4_quantize_flags_nonfinite():
    W = torch.zeros((1, 128, 256))
    W[0, 7, 9] = float("inf")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.int4_quantize(W.cuda(), dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & moe.DEVERR_NONFINITE


def _ragged(counts):
    off = np.zeros(len(counts) + 1, dtype=np.int32)
    off[1:] = np.cumsum(counts)
    return off


@pytest.mark.parametrize("epi", ["none", "swiglu"])
@pytest.mark.parametrize("counts", [[1, 0, 9, 16, 17, 40], [8, 8, 0, 3]])
def test_int4_grouped_gemm_ragged(epi, counts):
    E = len(counts)
    off = _ragged(counts)
    M = int(off[-1])
    g = torch.Generator().manual_seed(sum(counts) + len(epi))
    N, K = (256, 768) if epi == "swiglu" else (384, 512)
    W = torch.randn((E, N, K), generator=g) * 0.03
    X = torch.randn((M, K), generator=g).to(torch.float16)
    packed, meta = moe.int4_quantize(W.cuda())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = moe.int4_grouped_gemm(X.cuda(), packed, meta, torch.from_numpy(off).cuda(), M,
                                epilogue=epi, out_dtype=torch.float32, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    p_ref, m_ref = oracle.quantize_int4_grouped(W.numpy())
    ref = oracle.grouped_gemm_int4(X.float().numpy(), p_ref, m_ref, off)
    if epi == "swiglu":
        ref = oracle.swiglu(ref)
    assert_close(_np(out), ref, f"int4 {epi} {counts}")


@pytest.mark.parametrize("out_dtype", [torch.float16, torch.bfloat16])
def test_int4_grouped_gemm_output_dtypes(out_dtype):
    E, N, K = 2, 128, 256
    counts = [5, 12]
    off = _ragged(counts)
    M = int(off[-1])
    g = torch.Generator().manual_seed(7)
    W = torch.randn((E, N, K), generator=g) * 0.03
    X = torch.randn((M, K), generator=g).to(torch.float16)
    packed, meta = moe.int4_quantize(W.cuda())
    out = moe.int4_grouped_gemm(X.cuda(), packed, meta, torch.from_numpy(off).cuda(), M,
                                out_dtype=out_dtype)
    torch.cuda.synchronize()
    p_ref, m_ref = oracle.quantize_int4_grouped(W.numpy())
    ref = oracle.grouped_gemm_int4(X.float().numpy(), p_ref, m_ref, off)
    assert_close_16bit(out.double().cpu().numpy(), ref, out_dtype, f"int4 out {out_dtype}")


def test_int4_grouped_gemm_flags_bad_offsets():
    E, N, K = 2, 128, 256
    packed = torch.zeros((E, N, K // 2), dtype=torch.uint8, device="cuda")
    meta = torch.zeros((E, N, K // 128), dtype=torch.int32, device="cuda")
    X = torch.ones((8, K), dtype=torch.float16, device="cuda")
    bad = torch.tensor([0, 9, 8], dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.int4_grouped_gemm(X, packed, meta, bad, 8, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & moe.DEVERR_BAD_OFFSETS


@pytest.mark.parametrize("epi", ["none", "swiglu"])
@pytest.mark.parametrize("counts", [[1, 0, 15, 16, 17, 300], [0, 0, 513, 0, 2, 256]])
def test_int4_tc_grouped_gemm_ragged(epi, counts):
    # the tcgen05 kernel on INT4 weights, fp16((q - z) s) in tensor memory;
    # K = 384 has no decode-GEMV form
    off = _ragged(counts)
    E, M = len(counts), int(off[-1])
    g = torch.Generator().manual_seed(sum(counts) + 13 * len(epi))
    N, K = (512, 384) if epi == "swiglu" else (256, 640)
    W = torch.randn((E, N, K), generator=g) * 0.03
    X = torch.randn((M, K), generator=g).to(torch.float16)
    packed, meta = moe.int4_quantize(W.cuda())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = moe.int4_grouped_gemm(X.cuda(), packed, meta, torch.from_numpy(off).cuda(), M,
                                epilogue=epi, out_dtype=torch.float32, algo="tc", dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    p_ref, m_ref = oracle.quantize_int4_grouped(W.numpy())
    ref = oracle.grouped_gemm_int4(X.float().numpy(), p_ref, m_ref, off)
    if epi == "swiglu":
        ref = oracle.swiglu(ref)
    assert_close(out.cpu().numpy(), ref, f"int4 tc {epi} {counts}")


@pytest.mark.parametrize("N,K,epi", [(1536, 2048, "swiglu"), (2048, 768, "none")],
                         ids=["gate_up", "down"])
def test_int4_decode_at_qwen3_30b_projection_sizes(N, K, epi):
    # the decode pipeline's INT4 form at the Qwen3-30B-A3B projection sizes
    # (12 and 16 row tiles, 8 and 3 stages per item), three experts with 1, 0
    # and 19 routed rows (two items for the last)
    counts = [1, 0, 19]
    E = len(counts)
    off = _ragged(counts)
    M = int(off[-1])
    g = torch.Generator().manual_seed(N + K)
    W = torch.randn((E, N, K), generator=g) * 0.02
    X = torch.randn((M, K), generator=g).to(torch.float16)
    packed, meta = moe.int4_quantize(W.cuda())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = moe.int4_grouped_gemm(X.cuda(), packed, meta, torch.from_numpy(off).cuda(), M,
                                epilogue=epi, out_dtype=torch.float32, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    p_ref, m_ref = oracle.quantize_int4_grouped(W.numpy())
    ref = oracle.grouped_gemm_int4(X.float().numpy(), p_ref, m_ref, off)
    if epi == "swiglu":
        ref = oracle.swiglu(ref)
    assert_close(_np(out), ref, f"int4 30b {epi}")
