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
from parity_util import assert_close, assert_close_16bit

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


# ----------------------------------------------------------------- tensor cores

@pytest.mark.parametrize("counts,N,K", [([1, 0, 300, 33], 2048, 1024),   # two token tiles, an empty expert
                                        ([40, 257, 3], 192, 768),        # three reduction stages
                                        ([64], 64, 256)])                # one stage, two column tiles
@pytest.mark.parametrize("odt", [torch.float32, torch.float16])
def test_grouped_gemm_t_tensor_cores(counts, N, K, odt):
    # the tcgen05 kernel in its transposed form: each TMEM lane an output
    # column k, the reduction over the weight rows n
    E = len(counts)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(off[-1])
    g = torch.Generator().manual_seed(N + K + M + 1)
    W = torch.randn((E, N, K), generator=g) * 0.05
    G = torch.randn((M + 2, N), generator=g).to(torch.float16)
    p, a = moe.nf4_quantize(W.cuda())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = moe.nf4_grouped_gemm_t(G.cuda(), p, a, torch.from_numpy(off).cuda(), M, out_dtype=odt,
                                 dev_err=err, algo="tc")
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    P, S = oracle.quantize_blockwise(W.numpy())
    ref = bw.grouped_gemm_t(G[:M].double().numpy(), P, S.reshape(E, -1), off)
    if odt == torch.float32:
        assert_close(_np(out), ref, f"gemm_t tc {counts} {N} {K}")
    else:
        assert_close_16bit(_np(out.double()), ref, odt, f"gemm_t tc {counts} {N} {K}")


@pytest.mark.parametrize("odt", [torch.float32, torch.float16])
def test_down_backward_fused(odt):
    # transposed down GEMM and the SwiGLU backward in one launch
    counts = [5, 0, 290, 17]
    E, H, I = len(counts), 512, 256
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(off[-1])
    g = torch.Generator().manual_seed(77)
    W = torch.randn((E, H, I), generator=g) * 0.05
    dYp = torch.randn((M, H), generator=g).to(torch.float16)
    gu = torch.randn((M, 2 * I), generator=g) * 2
    p, a = moe.nf4_quantize(W.cuda())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    dgu = moe.nf4_down_backward(dYp.cuda(), p, a, torch.from_numpy(off).cuda(), M, gu.cuda(),
                                out_dtype=odt, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    P, S = oracle.quantize_blockwise(W.numpy())
    dh = bw.grouped_gemm_t(dYp.double().numpy(), P, S.reshape(E, -1), off)
    ref = bw.swiglu_backward(gu.double().numpy(), dh)
    if odt == torch.float32:
        assert_close(_np(dgu), ref, "down backward fused")
    else:
        assert_close_16bit(_np(dgu.double()), ref, odt, "down backward fused")


def test_layer_backward_qwen3_30b_prefill_tensor_cores():
    # The Qwen3-30B-A3B-shaped prefill layer (4096 tokens, Zipf routing):
    # forward with fp32 pre-activations, then combine backward (fp16 dYp) ->
    # transposed down + SwiGLU backward in one tensor-core launch -> transposed
    # gate_up on the tensor cores -> scatter-add -> routing backward; dx and
    # dlogits on 64 seeded tokens against the oracle (tokens are independent,
    # so the oracle runs on those tokens alone)
    import moe_synth
    from parity_util import LazyOracleStack, gpu_stack
    shape, T, seed = moe_synth.QWEN3_30B, 4096, 2
    stack_gpu, weights = gpu_stack(shape, seed)
    stack = LazyOracleStack.shared(stack_gpu, weights)
    p_gu, a_gu, p_d, a_d = stack_gpu
    x = moe_synth.activations(T, shape.H, seed)
    lg = moe_synth.logits(shape, T, seed)
    dY = torch.randn((T, shape.H), generator=torch.Generator().manual_seed(9))
    k, M = shape.k, T * shape.k
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    r = moe.route_permute(lg.cuda(), k, shape.renormalize)
    Xp = moe.permute_rows(x.cuda(), r["sorted_rows"], k)
    GU = moe.nf4_grouped_gemm(Xp, p_gu, a_gu, r["expert_offsets"], M, out_dtype=torch.float32)
    Hh = moe.swiglu(GU, h_dtype=torch.float16)
    Yp = moe.nf4_grouped_gemm(Hh, p_d, a_d, r["expert_offsets"], M, out_dtype=torch.float32)
    dYp, dw = moe.combine_backward(dY.cuda(), Yp, r["inv_perm"], r["topk_w"],
                                   dyp_dtype=torch.float16)
    dGU = moe.nf4_down_backward(dYp, p_d, a_d, r["expert_offsets"], M, GU,
                                out_dtype=torch.float16, dev_err=err)
    dXp = moe.nf4_grouped_gemm_t(dGU, p_gu, a_gu, r["expert_offsets"], M, algo="tc", dev_err=err)
    dx = moe.unpermute_combine(dXp, r["inv_perm"], torch.ones((T, k), device="cuda"))
    dl = moe.route_backward(lg.cuda(), r["topk_idx"], r["topk_w"], dw, shape.renormalize)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rng = np.random.default_rng(4)
    toks = sorted(rng.choice(T, size=64, replace=False).tolist())
    rdx, rdl, ridx, rdw = bw.moe_layer_backward(x.float().numpy()[toks], lg.numpy()[toks],
                                                stack, k, shape.renormalize,
                                                dY.double().numpy()[toks], with_dw=True)
    assert_close(_np(dx)[toks], rdx, "30b prefill dx (tensor cores)")
    _check_routing_grads(_np(r["topk_idx"])[toks], _np(dw)[toks], _np(dl)[toks], lg.numpy()[toks],
                         ridx, rdw, rdl, shape.renormalize, "30b prefill")


def _check_routing_grads(idx, dw, dl, logits, ridx, rdw, rdl, renorm, what):
    """The routing gradients of a layer backward, in three parts.

    dw (the gradient w.r.t. each selected expert's weight, dY . Yp) against
    the oracle's, matched by expert id.  dlogits against the oracle's routing
    backward applied to the GPU's own dw: that isolates the routing backward
    kernel.  And dlogits against the oracle end to end within the bound the
    routing backward's formula gives for an error in dw: with renormalisation
    dlogit_e = w_j (dw_j - sum_i w_i dw_i), so an error of at most d in every
    dw moves it by at most 2 w_j d <= 2 d (the softmax over all experts gives
    the same 2 d).  The subtraction there cancels most of dw when the experts'
    dw are alike, so the end-to-end comparison cannot use the relative bound:
    forward rounding (16-bit h) that is small against dw can be large against
    the difference."""
    T, k = idx.shape
    assert np.array_equal(np.sort(idx, axis=1), np.sort(ridx, axis=1)), f"{what}: selection"
    # the GPU's dw in the oracle's order of the selected experts
    order = np.array([[int(np.where(idx[t] == e)[0][0]) for e in ridx[t]] for t in range(T)])
    dw_o = np.take_along_axis(dw, order, axis=1)
    assert_close(dw_o, rdw, f"{what} dw")
    assert_close(dl, bw.route_backward(logits, ridx, dw_o, renorm),
                 f"{what} dlogits (oracle routing backward of the GPU's dw)")
    d = np.abs(dw_o - rdw).max(axis=1, keepdims=True)        # per token
    bound = 2.0 * d + 1e-6 * np.abs(rdl).max()
    excess = np.abs(dl - rdl) - bound
    assert np.all(excess <= 0), (f"{what} dlogits end to end: worst excess {excess.max():.3e} "
                                 f"over the bound from dw's error")
