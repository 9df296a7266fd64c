"""GPU parity of the backward kernels against ``oracle.backward``.

The backward kernels were first checked on a B200 through the C ABI alone
(``tests/c_abi``); this file checks them through the Python binding.  The
file name sorts after the forward-path GPU tests.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import backward as bw
from parity_util import assert_close

pytestmark = pytest.mark.gpu

moe = pytest.importorskip("bit_mixture_experts_route_b200")


def _np(t):
    return t.detach().cpu().numpy()


@pytest.mark.parametrize("counts,N,K", [([1, 0, 9, 3], 70, 320), ([8, 8, 0, 40], 2048, 1024),
                                        ([0, 17], 64, 64)])
@pytest.mark.parametrize("gdt", [torch.float32, torch.float16])
def test_grouped_gemm_t(counts, N, K, gdt):
    E = len(counts)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(off[-1])
    g = torch.Generator().manual_seed(N + K + M)
    W = torch.randn((E, N, K), generator=g) * 0.05
    G = torch.randn((M + 2, N), generator=g).to(gdt)
    p, a = moe.nf4_quantize(W.cuda())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = moe.nf4_grouped_gemm_t(G.cuda(), p, a, torch.from_numpy(off).cuda(), M, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    P, S = oracle.quantize_blockwise(W.numpy())
    ref = bw.grouped_gemm_t(G[:M].double().numpy(), P, S.reshape(E, -1), off)
    assert_close(_np(out), ref, f"gemm_t {counts} {N} {K} {gdt}")


def test_swiglu_backward():
    g = torch.Generator().manual_seed(3)
    gu = torch.randn((37, 2 * 96), generator=g) * 3
    dh = torch.randn((37, 96), generator=g)
    out = moe.swiglu_backward(gu.cuda(), dh.cuda())
    torch.cuda.synchronize()
    assert_close(_np(out), bw.swiglu_backward(gu.double().numpy(), dh.double().numpy()), "swiglu bw")


@pytest.mark.parametrize("renorm", [True, False])
def test_combine_and_route_backward(renorm):
    g = torch.Generator().manual_seed(5 + renorm)
    T, E, k, H = 33, 16, 4, 256
    lg = torch.randn((T, E), generator=g)
    r = moe.route_permute(lg.cuda(), k, renorm)
    Yp = torch.randn((T * k, H), generator=g)
    dY = torch.randn((T, H), generator=g)
    dYp, dw = moe.combine_backward(dY.cuda(), Yp.cuda(), r["inv_perm"], r["topk_w"])
    dl = moe.route_backward(lg.cuda(), r["topk_idx"], r["topk_w"], dw, renorm)
    torch.cuda.synchronize()
    idx, w = oracle.route_topk(lg.numpy(), k, renorm)
    _, _, inv = oracle.permute_by_expert(idx, E)
    rdYp, rdw = bw.combine_backward(dY.double().numpy(), Yp.double().numpy(), inv, w)
    assert_close(_np(dYp), rdYp, "combine bw dYp")
    assert_close(_np(dw), rdw, "combine bw dw")
    assert_close(_np(dl), bw.route_backward(lg.numpy(), idx, rdw, renorm), "route bw")


def test_layer_backward_through_the_kernels():
    # recompute forward (fp32 pre-activations), then combine bw -> transposed
    # down -> SwiGLU bw -> transposed gate_up -> scatter-add -> routing bw
    E, k, H, I, T = 8, 2, 256, 128, 24
    g = torch.Generator().manual_seed(11)
    w_gu = torch.randn((E, 2 * I, H), generator=g) * 0.05
    w_d = torch.randn((E, H, I), generator=g) * 0.05
    x = torch.randn((T, H), generator=g).to(torch.bfloat16)
    lg = torch.randn((T, E), generator=g)
    dY = torch.randn((T, H), generator=g)
    p_gu, a_gu = moe.nf4_quantize(w_gu.cuda())
    p_d, a_d = moe.nf4_quantize(w_d.cuda())
    r = moe.route_permute(lg.cuda(), k, True)
    M = T * k
    Xp = moe.permute_rows(x.cuda(), r["sorted_rows"], k)
    GU = moe.nf4_grouped_gemm(Xp, p_gu, a_gu, r["expert_offsets"], M, out_dtype=torch.float32)
    Hh = moe.swiglu(GU, h_dtype=torch.float16)
    Yp = moe.nf4_grouped_gemm(Hh, p_d, a_d, r["expert_offsets"], M, out_dtype=torch.float32)
    dYp, dw = moe.combine_backward(dY.cuda(), Yp, r["inv_perm"], r["topk_w"])
    dH = moe.nf4_grouped_gemm_t(dYp, p_d, a_d, r["expert_offsets"], M)
    dGU = moe.swiglu_backward(GU, dH)
    dXp = moe.nf4_grouped_gemm_t(dGU, p_gu, a_gu, r["expert_offsets"], M)
    ones = torch.ones((T, k), dtype=torch.float32, device="cuda")
    dx = moe.unpermute_combine(dXp, r["inv_perm"], ones)
    dl = moe.route_backward(lg.cuda(), r["topk_idx"], r["topk_w"], dw, True)
    torch.cuda.synchronize()
    P_gu, S_gu = oracle.quantize_blockwise(w_gu.numpy())
    P_d, S_d = oracle.quantize_blockwise(w_d.numpy())
    stack = oracle.ExpertStack(P_gu, S_gu.reshape(E, -1), P_d, S_d.reshape(E, -1))
    rdx, rdl = bw.moe_layer_backward(x.float().numpy(), lg.numpy(), stack, k, True,
                                     dY.double().numpy())
    assert_close(_np(dx), rdx, "layer dx")
    assert_close(_np(dl), rdl, "layer dlogits")
