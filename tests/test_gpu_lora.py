"""GPU parity of the per-expert LoRA delta (``moe_lora_delta``) against the
CPU oracle (``oracle.lora``), alone and composed with the 4-bit grouped GEMMs
into an adapted expert MLP."""

import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_close

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("bit_mixture_experts_route_b200")


def _np(t):
    return t.detach().cpu().numpy()


def _ragged(counts):
    off = np.zeros(len(counts) + 1, dtype=np.int32)
    off[1:] = np.cumsum(counts)
    return off


def _adapters(g, E, N, K, r):
    A = (torch.randn((E, r, K), generator=g) / K ** 0.5).to(torch.float16)
    B = (torch.randn((E, N, r), generator=g) * 0.15).to(torch.float16)
    return A, B


# short segments (8-row tiles, column splits), long ones (16-row tiles), an
# expert-count past one warp's scan, K off the 256 stride, N off 256, ranks 8..64
CASES = [
    ([1, 0, 9, 16, 17, 40], 300, 264, 8),
    ([8] * 8, 2048, 2048, 16),
    ([0, 0, 33], 512, 16, 64),
    ([1] * 8 + [0] * 120, 3072, 512, 16),
    ([100, 3, 0, 29], 704, 128, 24),
    ([40 + (e * 7) % 23 for e in range(40)], 1024, 768, 32),
]


@pytest.mark.parametrize("counts,N,K,r", CASES)
def test_lora_delta_ragged(counts, N, K, r):
    E = len(counts)
    off = _ragged(counts)
    M = int(off[-1])
    g = torch.Generator().manual_seed(M + N + K + r)
    X = torch.randn((M + 3, K), generator=g).to(torch.float16)    # A_rows > M_total
    A, B = _adapters(g, E, N, K, r)
    base = torch.randn((M, N), generator=g)
    scale = 32.0 / r
    delta_ref = oracle.lora_delta(X[:M].double().numpy(), off, A.double().numpy(),
                                  B.double().numpy(), scale)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    offs = torch.from_numpy(off).cuda()
    # in place on a pre-activation
    out = base.cuda()
    moe.lora_delta(X.cuda(), offs, A.cuda(), B.cuda(), scale, out, dev_err=err)
    # and alone (out starts at zero)
    only = torch.zeros((M, N), device="cuda")
    moe.lora_delta(X.cuda(), offs, A.cuda(), B.cuda(), scale, only, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert_close(_np(only), delta_ref, f"lora delta {counts[:6]} N={N} K={K} r={r}")
    assert_close(_np(out), base.double().numpy() + delta_ref, "lora in place")


def test_lora_delta_bad_offsets_leave_out_unchanged():
    E, N, K, r = 3, 256, 256, 16
    g = torch.Generator().manual_seed(11)
    X = torch.randn((12, K), generator=g).to(torch.float16).cuda()
    A, B = _adapters(g, E, N, K, r)
    base = torch.randn((12, N), generator=g).cuda()
    for off in ([0, 8, 4, 12], [1, 4, 8, 12], [0, 4, 8, 11]):
        out = base.clone()
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        moe.lora_delta(X, torch.tensor(off, dtype=torch.int32, device="cuda"), A.cuda(), B.cuda(),
                       1.0, out, M_total=12, dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) & moe.DEVERR_BAD_OFFSETS, off
        assert torch.equal(out, base), off


def test_lora_delta_empty_is_a_no_op():
    E, N, K, r = 2, 128, 64, 8
    A = torch.zeros((E, r, K), dtype=torch.float16, device="cuda")
    B = torch.zeros((E, N, r), dtype=torch.float16, device="cuda")
    out = torch.empty((0, N), device="cuda")
    moe.lora_delta(torch.empty((0, K), dtype=torch.float16, device="cuda"),
                   torch.zeros(E + 1, dtype=torch.int32, device="cuda"), A, B, 1.0, out)
    torch.cuda.synchronize()


@pytest.mark.parametrize("algo", ["gemv", "tc"])
def test_adapted_expert_mlp_nf4(algo):
    """gate_up (no epilogue, fp32) + LoRA -> SwiGLU -> down (fp32) + LoRA,
    against the oracle's grouped GEMM plus its LoRA delta at each projection."""
    counts = [8, 0, 5, 19, 8, 1, 12, 11] if algo == "gemv" else [70, 0, 33, 129, 64, 16, 80, 100]
    E, H, I, r = len(counts), 512, 256, 16
    off = _ragged(counts)
    M = int(off[-1])
    g = torch.Generator().manual_seed(M + r)
    W_gu = torch.randn((E, 2 * I, H), generator=g) * 0.05
    W_d = torch.randn((E, H, I), generator=g) * 0.05
    X = torch.randn((M, H), generator=g).to(torch.float16)
    A_gu, B_gu = _adapters(g, E, 2 * I, H, r)
    A_d, B_d = _adapters(g, E, H, I, r)
    scale = 2.0
    p_gu, a_gu = moe.nf4_quantize(W_gu.cuda())
    p_d, a_d = moe.nf4_quantize(W_d.cuda())
    offs = torch.from_numpy(off).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    gu = moe.nf4_grouped_gemm(X.cuda(), p_gu, a_gu, offs, M, epilogue="none",
                              out_dtype=torch.float32, algo=algo, dev_err=err)
    moe.lora_delta(X.cuda(), offs, A_gu.cuda(), B_gu.cuda(), scale, gu, dev_err=err)
    h = moe.swiglu(gu, h_dtype=torch.float16)
    y = moe.nf4_grouped_gemm(h, p_d, a_d, offs, M, epilogue="none", out_dtype=torch.float32,
                             algo=algo, dev_err=err)
    moe.lora_delta(h, offs, A_d.cuda(), B_d.cuda(), scale, y, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0

    P_gu, S_gu = oracle.quantize_blockwise(W_gu.numpy())
    P_d, S_d = oracle.quantize_blockwise(W_d.numpy())
    x = X.double().numpy()
    gu_ref = oracle.grouped_gemm(x, P_gu, S_gu.reshape(E, -1), off) + oracle.lora_delta(
        x, off, A_gu.double().numpy(), B_gu.double().numpy(), scale)
    h_ref = oracle.swiglu(gu_ref)
    y_ref = oracle.grouped_gemm(h_ref, P_d, S_d.reshape(E, -1), off) + oracle.lora_delta(
        h_ref, off, A_d.double().numpy(), B_d.double().numpy(), scale)
    assert_close(_np(gu), gu_ref, f"adapted gate_up ({algo})")
    assert_close(_np(y), y_ref, f"adapted expert MLP ({algo})")
