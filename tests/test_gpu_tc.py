"""GPU parity of the tensor-core (tcgen05) grouped NF4 GEMM and of the
activation permutation that feeds it, against the CPU oracle."""

import numpy as np
import pytest
import torch

import moe_synth
import oracle
from parity_util import LazyOracleStack, assert_close, gpu_stack

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("bit_mixture_experts_route_b200")


def _np(t):
    return t.detach().cpu().numpy()


def test_permute_rows_exact():
    g = torch.Generator().manual_seed(1)
    T, K, k = 37, 320, 3
    X = torch.randn((T, K), generator=g).to(torch.bfloat16)
    rows = torch.randperm(T * k, generator=g).to(torch.int32)
    Xp = moe.permute_rows(X.cuda(), rows.cuda(), k)
    ref = X[rows.long() // k].to(torch.float16)   # bf16 -> fp16 is exact here
    assert torch.equal(Xp.cpu(), ref)
    bad = rows.clone()
    bad[5] = T * k + 3
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    Xb = moe.permute_rows(X.cuda(), bad.cuda(), k, dev_err=err)
    assert int(err.item()) & moe.DEVERR_BAD_INDEX
    assert torch.all(Xb[5] == 0)


def _ragged(E, counts):
    off = np.zeros(E + 1, dtype=np.int32)
    off[1:] = np.cumsum(counts)
    return off


@pytest.mark.parametrize("algo", ["tc", "tc_pair"])
@pytest.mark.parametrize("epi", ["none", "swiglu"])
@pytest.mark.parametrize("counts", [
    [1, 0, 15, 16, 17, 300],          # partial N tiles, an empty expert, two token tiles
    [0, 0, 513, 0, 2, 256],           # three token tiles, exact 256 tile
])
def test_tc_grouped_gemm_ragged(epi, counts, algo):
    E = len(counts)
    counts = np.array(counts)
    off = _ragged(E, counts)
    M = int(off[-1])
    g = torch.Generator().manual_seed(int(counts.sum()))
    N, K = (512, 256) if epi == "swiglu" else (256, 384)
    W = torch.randn((E, N, K), generator=g) * 0.05
    X = (torch.randn((M, K), generator=g)).to(torch.float16)
    p, a = moe.nf4_quantize(W.cuda())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = moe.nf4_grouped_gemm(X.cuda(), p, a, torch.from_numpy(off).cuda(), M, epilogue=epi,
                               out_dtype=torch.float32, algo=algo, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    pr, ar = oracle.quantize_blockwise(W.numpy())
    ref = oracle.grouped_gemm(X.float().numpy(), pr, ar.reshape(E, -1), off)
    if epi == "swiglu":
        ref = oracle.swiglu(ref)
    assert_close(_np(out), ref, f"{algo} {epi}")


@pytest.mark.parametrize("K", [64, 192, 320])
def test_tc_short_and_odd_k(K):
    # K / 64 k-stages per tile: 1 (fewer than the four decoder groups), 3 and
    # 5 (odd, so a group's stages straddle tile boundaries)
    E, N = 3, 256
    counts = np.array([5, 0, 40])
    off = _ragged(E, counts)
    M = int(off[-1])
    g = torch.Generator().manual_seed(K)
    W = torch.randn((E, N, K), generator=g) * 0.05
    X = torch.randn((M, K), generator=g).to(torch.float16)
    p, a = moe.nf4_quantize(W.cuda())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for epi in ("none", "swiglu"):
        out = moe.nf4_grouped_gemm(X.cuda(), p, a, torch.from_numpy(off).cuda(), M, epilogue=epi,
                                   out_dtype=torch.float32, algo="tc", dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        pr, ar = oracle.quantize_blockwise(W.numpy())
        ref = oracle.grouped_gemm(X.float().numpy(), pr, ar.reshape(E, -1), off)
        if epi == "swiglu":
            ref = oracle.swiglu(ref)
        assert_close(_np(out), ref, f"tc K={K} {epi}")


@pytest.mark.parametrize("algo", ["tc", "tc_pair"])
@pytest.mark.parametrize("epi,N,K", [("swiglu", 3072, 4096), ("none", 4096, 1536)],
                         ids=["gate_up", "down"])
def test_tc_grouped_gemm_qwen3_235b_dims(epi, N, K, algo):
    # The Qwen3-235B-A22B expert projections (gate_up 4096 -> 2*1536 with the
    # SwiGLU epilogue, down 1536 -> 4096) on four experts with ragged row
    # counts: an empty expert, partial and full 256-row token tiles, weights
    # N(0, 0.015) with 0.1 % outliers at 8 sigma.
    counts = np.array([300, 0, 37, 256])
    E = len(counts)
    off = _ragged(E, counts)
    M = int(off[-1])
    g = torch.Generator().manual_seed(N + K)
    W = torch.randn((E, N, K), generator=g) * 0.015
    n_out = int(1e-3 * W.numel())
    pos = torch.randint(0, W.numel(), (n_out,), generator=g)
    W.view(-1)[pos] = 8 * 0.015 * torch.sign(torch.randn(n_out, generator=g))
    X = torch.randn((M, K), generator=g).to(torch.float16)
    p, a = moe.nf4_quantize(W.cuda())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = moe.nf4_grouped_gemm(X.cuda(), p, a, torch.from_numpy(off).cuda(), M, epilogue=epi,
                               out_dtype=torch.float32, algo=algo, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    pr, ar = oracle.quantize_blockwise(W.numpy())
    assert np.array_equal(_np(p), pr)
    ref = oracle.grouped_gemm(X.float().numpy(), pr, ar.reshape(E, -1), off)
    if epi == "swiglu":
        ref = oracle.swiglu(ref)
    assert_close(_np(out), ref, f"tc 235B {epi}")


def test_tc_flags_bad_offsets():
    E, N, K = 2, 128, 64
    p = torch.zeros((E, N, K // 2), dtype=torch.uint8, device="cuda")
    a = torch.ones((E, N * K // 64), dtype=torch.float32, device="cuda")
    X = torch.ones((8, K), dtype=torch.float16, device="cuda")
    bad = torch.tensor([0, 9, 8], dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.nf4_grouped_gemm(X, p, a, bad, 8, algo="tc", dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & moe.DEVERR_BAD_OFFSETS


def test_layer_qwen3_prefill_tc_sampled():
    shape, T, seed = moe_synth.QWEN3_30B, 4096, 2
    stack_gpu, weights = gpu_stack(shape, seed)
    stack = LazyOracleStack.shared(stack_gpu, weights)
    X = moe_synth.activations(T, shape.H, seed)
    lg = moe_synth.logits(shape, T, seed)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = moe.layer_forward(X.cuda(), lg.cuda(), shape.k, shape.renormalize, *stack_gpu,
                          dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rng = np.random.default_rng(1)
    toks = sorted(rng.choice(T, size=256, replace=False).tolist())
    ref = oracle.moe_layer(X.float().numpy(), lg.numpy(), stack, shape.k, shape.renormalize,
                           tokens=toks)
    assert_close(_np(Y)[toks], ref, "qwen3 prefill (tensor cores)")


@pytest.mark.parametrize("epi,N,K", [("none", 384, 256), ("swiglu", 640, 192)])
def test_tc_single_cta_form(epi, N, K):
    # N not a multiple of 256 (the pair form's tile): single-CTA tiles of 128
    # weight rows, and the pair form is refused
    counts = np.array([33, 0, 300, 7])
    E = len(counts)
    off = _ragged(E, counts)
    M = int(off[-1])
    g = torch.Generator().manual_seed(N + K + 1)
    W = torch.randn((E, N, K), generator=g) * 0.05
    X = torch.randn((M, K), generator=g).to(torch.float16)
    p, a = moe.nf4_quantize(W.cuda())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = moe.nf4_grouped_gemm(X.cuda(), p, a, torch.from_numpy(off).cuda(), M, epilogue=epi,
                               out_dtype=torch.float32, algo="tc", dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    pr, ar = oracle.quantize_blockwise(W.numpy())
    ref = oracle.grouped_gemm(X.float().numpy(), pr, ar.reshape(E, -1), off)
    if epi == "swiglu":
        ref = oracle.swiglu(ref)
    assert_close(_np(out), ref, f"tc single-CTA {epi}")
    with pytest.raises(moe.MoEError, match="UNSUPPORTED"):
        moe.nf4_grouped_gemm(X.cuda(), p, a, torch.from_numpy(off).cuda(), M, epilogue=epi,
                             algo="tc_pair")


@pytest.mark.parametrize("counts", [[1, 2, 3, 31, 32, 33], [255, 257, 1, 0, 0, 64]])
def test_tc_pair_form_small_and_odd_tiles(counts):
    # the pair form rounds a tile's routed rows up to 32 and splits them
    # between the two CTAs: tiles of 1..33 rows and tiles straddling 256
    E = len(counts)
    counts = np.array(counts)
    off = _ragged(E, counts)
    M = int(off[-1])
    g = torch.Generator().manual_seed(int(counts.sum()) + 5)
    N, K = 512, 320
    W = torch.randn((E, N, K), generator=g) * 0.05
    X = torch.randn((M, K), generator=g).to(torch.float16)
    p, a = moe.nf4_quantize(W.cuda())
    pr, ar = oracle.quantize_blockwise(W.numpy())
    ref = oracle.grouped_gemm(X.float().numpy(), pr, ar.reshape(E, -1), off)
    for epi in ("none", "swiglu"):
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = moe.nf4_grouped_gemm(X.cuda(), p, a, torch.from_numpy(off).cuda(), M, epilogue=epi,
                                   out_dtype=torch.float32, algo="tc_pair", dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        r = oracle.swiglu(ref) if epi == "swiglu" else ref
        assert_close(_np(out), r, f"tc pair {epi} {counts.tolist()}")
