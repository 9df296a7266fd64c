"""GPU parity of the MXFP4 path (quantize bit-exact, decode GEMV and
tensor-core GEMM within tolerance) against the CPU oracle (``oracle.mxfp4``).

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


# ----------------------------------------------------------------- tensor cores

@pytest.mark.parametrize("epi", ["none", "swiglu"])
@pytest.mark.parametrize("counts", [[1, 0, 15, 16, 17, 300], [0, 0, 513, 0, 2, 256]])
def test_mxfp4_tc_grouped_gemm_ragged(epi, counts):
    # the tcgen05 kernel on MXFP4 weights: partial and multiple 256-row token
    # tiles, empty experts, K off the GEMV's 256 stride (320)
    E = len(counts)
    off = _ragged(counts)
    M = int(off[-1])
    g = torch.Generator().manual_seed(sum(counts) + 7 * len(epi))
    N, K = (512, 320) if epi == "swiglu" else (256, 384)
    W = torch.randn((E, N, K), generator=g) * 0.03
    X = torch.randn((M, K), generator=g).to(torch.float16)
    packed, scales = moe.mxfp4_quantize(W.cuda())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = moe.mxfp4_grouped_gemm(X.cuda(), packed, scales, torch.from_numpy(off).cuda(), M,
                                 epilogue=epi, out_dtype=torch.float32, algo="tc", dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    p_ref, s_ref = oracle.quantize_mxfp4(W.numpy())
    ref = oracle.grouped_gemm_mxfp4(X.float().numpy(), p_ref, s_ref, off)
    if epi == "swiglu":
        ref = oracle.swiglu(ref)
    assert_close(_np(out), ref, f"mxfp4 tc {epi} {counts}")


def test_mxfp4_tc_scale_out_of_exact_range_is_flagged():
    E, N, K = 1, 128, 256
    off = _ragged([40])
    W = torch.randn((E, N, K)) * 0.05
    packed, scales = moe.mxfp4_quantize(W.cuda())
    scales[0, 0, 0] = 150                                 # 2^23: products overflow fp16
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.mxfp4_grouped_gemm(torch.zeros((40, K), dtype=torch.float16, device="cuda"), packed,
                           scales, torch.from_numpy(off).cuda(), 40, algo="tc", dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & moe.DEVERR_RANGE


def test_mxfp4_layer_qwen3_30b_prefill_tc_sampled():
    # The Qwen3-30B-A3B-shaped prefill (4096 tokens, Zipf routing) on MXFP4
    # experts through the exported calls: route, permute, gate_up + SwiGLU and
    # down on the tensor cores (AUTO at 256 rows per expert on average),
    # combine; 64 seeded tokens against the oracle's MXFP4 layer.
    import moe_synth
    shape, T, seed = moe_synth.QWEN3_30B, 4096, 6
    w_gu = moe_synth.weights(shape, "gate_up", seed, device="cuda")
    w_d = moe_synth.weights(shape, "down", seed, device="cuda")
    p_gu, s_gu = moe.mxfp4_quantize(w_gu)
    p_d, s_d = moe.mxfp4_quantize(w_d)
    X = moe_synth.activations(T, shape.H, seed)
    lg = moe_synth.logits(shape, T, seed)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    r = moe.route_permute(lg.cuda(), shape.k, shape.renormalize)
    M = T * shape.k
    Xp = moe.permute_rows(X.cuda(), r["sorted_rows"], shape.k)
    Hh = moe.mxfp4_grouped_gemm(Xp, p_gu, s_gu, r["expert_offsets"], M, epilogue="swiglu",
                                out_dtype=torch.float16, dev_err=err)
    Yp = moe.mxfp4_grouped_gemm(Hh, p_d, s_d, r["expert_offsets"], M, out_dtype=torch.float16,
                                dev_err=err)
    Y = moe.unpermute_combine(Yp, r["inv_perm"], r["topk_w"])
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rng = np.random.default_rng(3)
    toks = sorted(rng.choice(T, size=64, replace=False).tolist())
    idx, _ = oracle.route_topk(lg.numpy(), shape.k, shape.renormalize)
    experts = sorted({int(e) for t in toks for e in idx[t]})
    E, I, H = shape.E, shape.I, shape.H
    pg = np.zeros((E, 2 * I, H // 2), np.uint8)
    sg = np.zeros((E, 2 * I, H // 32), np.uint8)
    pd = np.zeros((E, H, I // 2), np.uint8)
    sd = np.zeros((E, H, I // 32), np.uint8)
    for e in experts:   # the oracle quantizes the experts it needs and checks the GPU's bytes
        pg[e], sg[e] = oracle.quantize_mxfp4(w_gu[e].cpu().numpy())
        pd[e], sd[e] = oracle.quantize_mxfp4(w_d[e].cpu().numpy())
        assert np.array_equal(_np(p_gu[e]), pg[e]) and np.array_equal(_np(s_gu[e]), sg[e])
        assert np.array_equal(_np(p_d[e]), pd[e]) and np.array_equal(_np(s_d[e]), sd[e])
    stack = oracle.Mxfp4ExpertStack(pg, sg, pd, sd)
    ref = oracle.moe_layer(X.float().numpy(), lg.numpy(), stack, shape.k, shape.renormalize,
                           tokens=toks)
    assert_close(_np(Y)[toks], ref, "mxfp4 qwen3-30b prefill (tensor cores)")


@pytest.mark.parametrize("N,K,epi", [(1536, 2048, "swiglu"), (2048, 768, "none")],
                         ids=["gate_up", "down"])
def test_mxfp4_decode_at_qwen3_30b_projection_sizes(N, K, epi):
    # the decode pipeline's MXFP4 form at the Qwen3-30B-A3B projection sizes
    # (12 and 16 row tiles, 8 and 3 stages per item), three experts with 1, 0
    # and 19 routed rows (two items for the last)
    counts = [1, 0, 19]
    E = len(counts)
    off = _ragged(counts)
    M = int(off[-1])
    g = torch.Generator().manual_seed(N + K + 1)
    W = torch.randn((E, N, K), generator=g) * 0.02
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
    assert_close(_np(out), ref, f"mxfp4 30b {epi}")
