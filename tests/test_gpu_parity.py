"""GPU parity: every exported call of libmoenf4.so against the CPU oracle.

Bit-exact: NF4 codes, absmax, top-k indices, expert offsets, sorted rows,
inverse permutation.  Floating point: routing weights to 2e-6 relative; the
GEMM, SwiGLU, combine and layer outputs within rel_max <= 1e-2 and
mae <= 1e-3 * RMS (tests/parity_util.py).
"""

import numpy as np
import pytest
import torch

import moe_synth
import oracle
from parity_util import (LazyOracleStack, assert_close, assert_close_16bit, gpu_stack,
                         run_layer_steps)

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("bit_mixture_experts_route_b200")


def _np(t):
    return t.detach().cpu().numpy()


# ----------------------------------------------------------------- NF4 table

def test_gpu_codebook_is_the_oracle_codebook():
    codes = np.arange(16, dtype=np.uint8)
    packed = torch.zeros((1, 1, 32), dtype=torch.uint8)
    b = (codes[0::2] << 4) | codes[1::2]
    packed[0, 0, :8] = torch.from_numpy(b)
    packed[0, 0, 8:] = 0x77
    absmax = torch.ones((1, 1), dtype=torch.float32)
    got = _np(moe.nf4_dequantize(packed.cuda(), absmax.cuda()))[0, 0, :16]
    assert np.array_equal(got.view(np.int32), oracle.nf4_levels().view(np.int32))


# ----------------------------------------------------------------- quantize

@pytest.mark.parametrize("E,N,K,sigma,outliers", [
    (8, 1024, 256, 0.02, 0.0),      # tiny gate_up
    (3, 256, 2048, 0.015, 1e-3),    # 235B-like with 8-sigma outliers
    (2, 64, 64, 1.0, 0.0),          # one block per row
])
def test_quantize_bit_exact(E, N, K, sigma, outliers):
    g = torch.Generator().manual_seed(E * 7 + K)
    W = torch.randn((E, N, K), generator=g) * sigma
    if outliers:
        n = int(outliers * W.numel())
        pos = torch.randint(0, W.numel(), (n,), generator=g)
        W.view(-1)[pos] = 8 * sigma * torch.sign(torch.randn(n, generator=g))
    W[0, 0, :64] = 0.0                       # an all-zero block
    W[0, 1, :16] = W[0, 1, 0]                # repeated maxima
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    p, a = moe.nf4_quantize(W.cuda(), dev_err=err)
    pr, ar = oracle.quantize_blockwise(W.numpy())
    assert p.numel() > 0
    assert np.array_equal(_np(p), pr)
    assert np.array_equal(_np(a).view(np.int32), ar.reshape(E, -1).view(np.int32))
    assert int(err.item()) == 0


def test_quantize_midpoint_ties_bit_exact():
    M = oracle.nf4_midpoints()
    W = np.zeros((1, 4, 64), dtype=np.float32)
    W[0, :, 0] = 1.0
    W[0, 0, 1:16] = M                          # exactly on each midpoint
    W[0, 1, 1:16] = np.nextafter(M, np.float32(2))   # just above
    W[0, 2, 1:16] = np.nextafter(M, np.float32(-2))  # just below
    W[0, 3, 1:17] = oracle.nf4_levels()        # exactly on each level
    p, a = moe.nf4_quantize(torch.from_numpy(W).cuda())
    pr, ar = oracle.quantize_blockwise(W)
    assert np.array_equal(_np(p), pr)
    assert np.array_equal(_np(a), ar.reshape(1, -1))


def test_quantize_flags_nonfinite():
    W = torch.zeros((1, 64, 128), device="cuda")
    W[0, 5, 7] = float("nan")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.nf4_quantize(W, dev_err=err)
    assert int(err.item()) & moe.DEVERR_NONFINITE


def test_quantize_negative_control():
    # The bit-exact gate must be able to fail: flip one nibble of the
    # oracle's expected codes and the comparison no longer holds.
    W = torch.randn((1, 64, 128), generator=torch.Generator().manual_seed(3))
    p, _ = moe.nf4_quantize(W.cuda())
    pr, _ = oracle.quantize_blockwise(W.numpy())
    pr[0, 3, 5] ^= 0x01
    assert not np.array_equal(_np(p), pr)


# ----------------------------------------------------------------- routing

def _route_case(shape, T, seed, logits=None, renorm=None):
    lg = moe_synth.logits(shape, T, seed) if logits is None else logits
    renorm = shape.renormalize if renorm is None else renorm
    r = moe.route_permute(lg.cuda(), shape.k, renorm)
    idx, w = oracle.route_topk(lg.numpy(), shape.k, renorm)
    off, rows, inv = oracle.permute_by_expert(idx, shape.E)
    assert np.array_equal(_np(r["topk_idx"]), idx)
    assert np.array_equal(_np(r["expert_offsets"]), off)
    assert np.array_equal(_np(r["sorted_rows"]), rows)
    assert np.array_equal(_np(r["inv_perm"]), inv)
    if T:
        np.testing.assert_allclose(_np(r["topk_w"]), w, rtol=2e-6, atol=1e-9)
    return r


@pytest.mark.parametrize("name,T", [("tiny", 16), ("olmoe", 1), ("olmoe", 64),
                                    ("qwen3-30b-a3b", 64), ("qwen3-30b-a3b", 4096),
                                    ("qwen3-235b-a22b", 2048), ("tiny", 0), ("olmoe", 131)])
def test_route_permute_bit_exact(name, T):
    _route_case(moe_synth.SHAPES[name], T, 0)


def test_route_ties_and_signed_zero():
    shape = moe_synth.MoEShape("ties", E=40, k=6, H=64, I=64, renormalize=True)
    g = torch.Generator().manual_seed(5)
    lg = torch.round(torch.randn((70, 40), generator=g) * 2) / 2
    lg[0] = 0.0
    lg[1, ::2] = -0.0
    _route_case(shape, 70, 0, logits=lg)


@pytest.mark.parametrize("E,k", [(1, 1), (8, 8), (256, 32), (1000, 4)])
def test_route_extreme_shapes(E, k):
    shape = moe_synth.MoEShape("x", E=E, k=k, H=64, I=64, renormalize=True)
    _route_case(shape, 33, E + k)
    _route_case(shape, 33, E + k, renorm=False)


def test_route_all_tokens_one_expert():
    shape = moe_synth.MoEShape("hot", E=16, k=2, H=64, I=64, renormalize=True)
    lg = torch.randn((200, 16), generator=torch.Generator().manual_seed(1))
    lg[:, 3] = 50.0
    r = _route_case(shape, 200, 0, logits=lg)
    off = _np(r["expert_offsets"])
    assert off[4] - off[3] == 200


# ----------------------------------------------------------------- GEMM

def _ragged_offsets(E, counts):
    off = np.zeros(E + 1, dtype=np.int32)
    off[1:] = np.cumsum(counts)
    return off


@pytest.mark.parametrize("algo", ["gemv"])
@pytest.mark.parametrize("epi", ["swiglu", "none"])
def test_grouped_gemm_ragged(algo, epi):
    # Experts with 0, 1, 7, 8, 9, 16, 17, 40 rows: empty experts, partial
    # and multiple 8-row MMA tiles, several 16-row chunks.
    E, H, I = 8, 256, 192
    counts = np.array([3, 0, 17, 1, 40, 8, 16, 9])
    off = _ragged_offsets(E, counts)
    M = int(off[-1])
    g = torch.Generator().manual_seed(11)
    N, K = (2 * I, H) if epi == "swiglu" else (H, I)
    W = torch.randn((E, N, K), generator=g) * 0.05
    p, a = moe.nf4_quantize(W.cuda())
    pr, ar = oracle.quantize_blockwise(W.numpy())
    if epi == "swiglu":
        T, k = 32, 3
        X = torch.randn((T, K), generator=g).to(torch.bfloat16)
        gather = torch.randperm(M, generator=g).to(torch.int32)
        out = moe.nf4_grouped_gemm(X.cuda(), p, a, torch.from_numpy(off).cuda(), M,
                                   gather=gather.cuda(), k=k, epilogue="swiglu",
                                   out_dtype=torch.float32, algo=algo)
        GU = oracle.grouped_gemm(X.float().numpy(), pr, ar.reshape(E, -1), off,
                                 gather=gather.numpy(), k=k)
        ref = oracle.swiglu(GU)
    else:
        X = (torch.randn((M, K), generator=g) * 0.3).to(torch.float16)
        out = moe.nf4_grouped_gemm(X.cuda(), p, a, torch.from_numpy(off).cuda(), M,
                                   epilogue="none", out_dtype=torch.float32, algo=algo)
        ref = oracle.grouped_gemm(X.float().numpy(), pr, ar.reshape(E, -1), off)
    assert_close(_np(out), ref, f"grouped gemm {epi}")


@pytest.mark.parametrize("out_dtype", [torch.float16, torch.bfloat16])
def test_grouped_gemm_output_dtypes(out_dtype):
    E, N, K = 4, 128, 128
    counts = np.array([5, 0, 12, 3])
    off = _ragged_offsets(E, counts)
    M = int(off[-1])
    g = torch.Generator().manual_seed(2)
    W = torch.randn((E, N, K), generator=g) * 0.05
    X = torch.randn((M, K), generator=g).to(torch.bfloat16)
    p, a = moe.nf4_quantize(W.cuda())
    out = moe.nf4_grouped_gemm(X.cuda(), p, a, torch.from_numpy(off).cuda(), M,
                               out_dtype=out_dtype)
    pr, ar = oracle.quantize_blockwise(W.numpy())
    ref = oracle.grouped_gemm(X.float().numpy(), pr, ar.reshape(E, -1), off)
    # A 16-bit output carries its own rounding (bf16: up to 2^-9 relative).
    # It must meet the bar against the unrounded oracle (that rounding counted
    # as error) and against the oracle rounded once to the output type.
    assert_close_16bit(_np(out.double()), ref, out_dtype, str(out_dtype))
    assert out.dtype == out_dtype


def test_grouped_gemm_flags_bad_offsets():
    E, N, K = 4, 64, 64
    p = torch.zeros((E, N, K // 2), dtype=torch.uint8, device="cuda")
    a = torch.ones((E, N * K // 64), dtype=torch.float32, device="cuda")
    X = torch.ones((8, K), dtype=torch.bfloat16, device="cuda")
    bad = torch.tensor([0, 5, 3, 8, 8], dtype=torch.int32, device="cuda")  # not monotone
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.nf4_grouped_gemm(X, p, a, bad, 8, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & moe.DEVERR_BAD_OFFSETS
    total_bad = torch.tensor([0, 2, 4, 6, 7], dtype=torch.int32, device="cuda")  # != M
    err.zero_()
    moe.nf4_grouped_gemm(X, p, a, total_bad, 8, dev_err=err)
    assert int(err.item()) & moe.DEVERR_BAD_OFFSETS


def test_grouped_gemm_flags_bad_gather():
    E, N, K = 2, 128, 64
    p = torch.zeros((E, N, K // 2), dtype=torch.uint8, device="cuda")
    a = torch.ones((E, N * K // 64), dtype=torch.float32, device="cuda")
    X = torch.ones((4, K), dtype=torch.bfloat16, device="cuda")
    off = torch.tensor([0, 2, 4], dtype=torch.int32, device="cuda")
    gather = torch.tensor([0, 1, 2, 99], dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.nf4_grouped_gemm(X, p, a, off, 4, gather=gather, k=1, epilogue="swiglu", dev_err=err)
    assert int(err.item()) & moe.DEVERR_BAD_INDEX


# ----------------------------------------------------------------- elementwise

@pytest.mark.parametrize("dt", [torch.float32, torch.float16])
def test_swiglu(dt):
    g = torch.Generator().manual_seed(4)
    gu = (torch.randn((37, 2 * 96), generator=g) * 3).to(dt)
    h = moe.swiglu(gu.cuda(), h_dtype=torch.float32)
    assert_close(_np(h), oracle.swiglu(gu.float().numpy()), "swiglu")


def test_combine():
    g = torch.Generator().manual_seed(6)
    T, k, H = 19, 4, 256
    Yp = torch.randn((T * k, H), generator=g)
    inv = torch.randperm(T * k, generator=g).to(torch.int32)
    w = torch.softmax(torch.randn((T, k), generator=g), 1)
    Y = moe.unpermute_combine(Yp.cuda(), inv.cuda(), w.cuda())
    ref = oracle.unpermute_combine(Yp.numpy(), inv.numpy(), w.numpy())
    assert_close(_np(Y), ref, "combine")


# ----------------------------------------------------------------- whole layer

def _layer_parity(shape, T, seed, tokens=None, algo="auto", via_layer_call=False):
    """The layer on seeded inputs against the oracle on ``tokens`` (all by
    default).  ``via_layer_call=False`` runs the exported calls one by one with
    the gate_up GEMM gathering its rows (``sorted_rows``): that always takes the
    general GEMV kernel.  ``via_layer_call=True`` runs ``moe_layer_forward``,
    which permutes the rows first and lets the AUTO rule pick the decode GEMV
    or, from 36 routed rows per expert on average, the tensor-core kernel."""
    stack_gpu, weights = gpu_stack(shape, seed)
    stack = LazyOracleStack.shared(stack_gpu, weights)
    X = moe_synth.activations(T, shape.H, seed)
    lg = moe_synth.logits(shape, T, seed)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    if via_layer_call:
        Y = moe.layer_forward(X.cuda(), lg.cuda(), shape.k, shape.renormalize, *stack_gpu,
                              dev_err=err)
    else:
        Y, *_ = run_layer_steps(X.cuda(), lg.cuda(), shape.k, shape.renormalize, stack_gpu,
                                algo=algo)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    toks = list(range(T)) if tokens is None else tokens
    ref = oracle.moe_layer(X.float().numpy(), lg.numpy(), stack, shape.k, shape.renormalize,
                           tokens=toks)
    assert stack.checked > 0
    return assert_close(_np(Y)[toks], ref, f"{shape.name} T={T}")


def _sample(T, n, seed):
    rng = np.random.default_rng(seed)
    return sorted(rng.choice(T, size=min(n, T), replace=False).tolist())


def test_layer_tiny_all_tokens():
    _layer_parity(moe_synth.TINY, 16, 0)


def test_layer_tiny_single_call():
    _layer_parity(moe_synth.TINY, 16, 0, via_layer_call=True)


@pytest.mark.parametrize("T", [1, 4, 16, 64])
def test_layer_olmoe_decode(T):
    _layer_parity(moe_synth.OLMOE, T, 0)


@pytest.mark.parametrize("T", [1, 4, 16, 64])
def test_layer_olmoe_decode_single_call(T):
    # the bench's layer: permuted rows, decode GEMV (TMA + warp MMA)
    _layer_parity(moe_synth.OLMOE, T, 0, via_layer_call=True)


def test_layer_olmoe_decode_last_layer():
    # layer 15 of the 16-layer decode stack (its own weights and logits)
    _layer_parity(moe_synth.OLMOE, 16, 15)


# Qwen3-30B-A3B-shaped decode, Zipf routing: the token sweep 1..64, all tokens
@pytest.mark.parametrize("T", [1, 2, 4, 8, 16, 32, 64])
def test_layer_qwen3_30b_decode_sweep(T):
    _layer_parity(moe_synth.QWEN3_30B, T, 1, via_layer_call=True)


def test_layer_qwen3_30b_decode_gather_path():
    _layer_parity(moe_synth.QWEN3_30B, 64, 1)


def test_layer_qwen3_30b_decode_last_layer():
    # layer 47 of the 48-layer decode stack
    _layer_parity(moe_synth.QWEN3_30B, 8, 47, via_layer_call=True)


def test_layer_qwen3_30b_prefill_gather_path_sampled():
    # 4096 tokens, Zipf routing (0 to ~1500 rows per expert, empty experts
    # included), through the gathering calls: both grouped GEMMs run on the
    # general GEMV kernel.  The tensor-core form of this layer is checked in
    # test_gpu_tc.py.
    _layer_parity(moe_synth.QWEN3_30B, 4096, 2, tokens=_sample(4096, 128, 0))


# Qwen3-235B-A22B-shaped layer: hidden 4096, moe_intermediate 1536, weights
# N(0, 0.015) with 0.1 % at 8 sigma.  Every case uses the weights of seed 3,
# so the oracle quantizes and checks each expert once for all of them.
_S235 = 3


@pytest.mark.parametrize("T", [1, 8, 32])
def test_layer_qwen3_235b_decode(T):
    _layer_parity(moe_synth.QWEN3_235B, T, _S235, via_layer_call=True)


@pytest.mark.parametrize("T", [8, 32])
def test_layer_qwen3_235b_decode_zipf(T):
    _layer_parity(moe_synth.QWEN3_235B_ZIPF, T, _S235, via_layer_call=True)


def test_layer_qwen3_235b_decode_gather_path():
    _layer_parity(moe_synth.QWEN3_235B, 8, _S235)


@pytest.mark.parametrize("shape", [moe_synth.QWEN3_235B, moe_synth.QWEN3_235B_ZIPF],
                         ids=["uniform", "zipf"])
def test_layer_qwen3_235b_prefill_tc_sampled(shape):
    # 2048 tokens (16384 routed rows, 128 per expert on average): the one-call
    # layer runs both grouped GEMMs on the tensor-core kernel; 128 seeded
    # tokens are checked against the oracle
    _layer_parity(shape, 2048, _S235, tokens=_sample(2048, 128, 1), via_layer_call=True)


def test_layer_single_expert_dense():
    shape = moe_synth.MoEShape("e1", E=1, k=1, H=256, I=128, renormalize=True, sigma=0.05)
    _layer_parity(shape, 9, 4)


def test_layer_deterministic():
    shape = moe_synth.TINY
    stack_gpu, _ = gpu_stack(shape, 0)
    X = moe_synth.activations(16, shape.H, 0).cuda()
    lg = moe_synth.logits(shape, 16, 0).cuda()
    y1 = moe.layer_forward(X, lg, shape.k, shape.renormalize, *stack_gpu)
    y2 = moe.layer_forward(X, lg, shape.k, shape.renormalize, *stack_gpu)
    assert torch.equal(y1, y2)


# ----------------------------------------------------------------- range guards

def _range_case(sigma_w, x_scale, epi, seed):
    E, K = 3, 256
    N = 512 if epi == "swiglu" else 256
    counts = np.array([5, 0, 40])
    off = _ragged_offsets(E, counts)
    M = int(off[-1])
    g = torch.Generator().manual_seed(seed)
    W = torch.randn((E, N, K), generator=g) * sigma_w
    X = (torch.randn((M, K), generator=g) * x_scale).to(torch.float16)
    p, a = moe.nf4_quantize(W.cuda())
    pr, ar = oracle.quantize_blockwise(W.numpy())
    ref = oracle.grouped_gemm(X.float().numpy(), pr, ar.reshape(E, -1), off)
    if epi == "swiglu":
        ref = oracle.swiglu(ref)
    return X.cuda(), p, a, torch.from_numpy(off).cuda(), M, ref


@pytest.mark.parametrize("algo", ["gemv", "tc"])
def test_range_tiny_weights(algo):
    # Weights ~N(0, 1e-5): every absmax lies below fp16's smallest normal
    # (2^-14).  The GEMV kernels apply the fp32 absmax to fp32 partial sums and
    # stay exact; the tensor-core kernel feeds fp16(level * absmax) and must
    # say so with MOE_DEVERR_RANGE.
    X, p, a, off, M, ref = _range_case(1e-5, 1.0, "none", 21)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = moe.nf4_grouped_gemm(X, p, a, off, M, out_dtype=torch.float32, algo=algo, dev_err=err)
    torch.cuda.synchronize()
    if algo == "gemv":
        assert int(err.item()) == 0
        assert_close(_np(out), ref, "gemv, weights 1e-5")
    else:
        assert int(err.item()) == moe.DEVERR_RANGE


@pytest.mark.parametrize("algo", ["gemv", "tc"])
def test_range_large_activations(algo):
    # Activations x 1e3 (fp16 holds them): fp32 and fp16 outputs in range meet
    # the bar with no flag on both kernels.
    X, p, a, off, M, ref = _range_case(0.02, 1e3, "none", 22)
    assert float(np.max(np.abs(ref))) < 6e4
    for dt in (torch.float32, torch.float16):
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = moe.nf4_grouped_gemm(X, p, a, off, M, out_dtype=dt, algo=algo, dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        if dt == torch.float32:
            assert_close(_np(out), ref, f"{algo}, x 1e3")
        else:
            assert_close_16bit(_np(out.double()), ref, dt, f"{algo}, x 1e3")


@pytest.mark.parametrize("algo", ["gemv", "tc"])
def test_range_fp16_output_overflow_flagged(algo):
    # x 1e3 activations through gate_up + SwiGLU: h = silu(g) * u reaches
    # ~1e5, beyond fp16.  An fp32 output is exact and unflagged; an fp16
    # output overflows and sets MOE_DEVERR_RANGE.
    X, p, a, off, M, ref = _range_case(0.05, 1e3, "swiglu", 23)
    assert float(np.max(np.abs(ref))) > 7e4
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = moe.nf4_grouped_gemm(X, p, a, off, M, epilogue="swiglu", out_dtype=torch.float32,
                               algo=algo, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert_close(_np(out), ref, f"{algo} swiglu fp32, x 1e3")
    out16 = moe.nf4_grouped_gemm(X, p, a, off, M, epilogue="swiglu", out_dtype=torch.float16,
                                 algo=algo, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == moe.DEVERR_RANGE
    assert torch.isinf(out16).any()


def test_range_permute_rows_overflow_flagged():
    # bf16 activations beyond fp16's range become inf in the fp16 rows the
    # grouped GEMMs read, and the call says so.
    T, K, k = 9, 256, 2
    X = torch.randn((T, K)).to(torch.bfloat16)
    X[4, 17] = 1e5
    rows = torch.arange(T * k, dtype=torch.int32)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    Xp = moe.permute_rows(X.cuda(), rows.cuda(), k, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == moe.DEVERR_RANGE
    assert torch.isinf(Xp[8, 17]) and torch.isinf(Xp[9, 17])
    err.zero_()
    moe.permute_rows((X * 0.5).clamp(-100, 100).cuda(), rows.cuda(), k, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
