"""Pins for the oracle's MoE layer (CPU only).

Three formulations of the layer -- per token and expert, the dense all-experts
brute force, and the explicit route/permute/grouped-GEMM/combine pipeline --
must agree; E = 1, k = 1 reduces to a dense SwiGLU MLP checked against
torch.nn.functional; planted mistakes (transposed weights, swapped gate/up,
a dropped combine weight) must fail.
"""

import numpy as np
import pytest
import torch

import moe_synth
import oracle


def _stack(shape, seed):
    wgu = moe_synth.weights(shape, "gate_up", seed).numpy()
    wd = moe_synth.weights(shape, "down", seed).numpy()
    pgu, agu = oracle.quantize_blockwise(wgu)
    pd, ad = oracle.quantize_blockwise(wd)
    return oracle.ExpertStack(pgu, agu.reshape(shape.E, -1), pd, ad.reshape(shape.E, -1))


MICRO = moe_synth.MoEShape("micro", E=4, k=2, H=64, I=64, renormalize=True, sigma=0.1)


@pytest.mark.parametrize("shape,T", [(moe_synth.TINY, 16), (MICRO, 4)])
def test_three_formulations_agree(shape, T):
    stack = _stack(shape, 0)
    x = moe_synth.activations(T, shape.H, 0).float().numpy()
    lg = moe_synth.logits(shape, T, 0).numpy()
    y1 = oracle.moe_layer(x, lg, stack, shape.k, shape.renormalize)
    y2 = oracle.moe_layer_dense(x, lg, stack, shape.k, shape.renormalize)
    y3 = oracle.moe_layer_permuted(x, lg, stack, shape.k, shape.renormalize)
    scale = np.sqrt(np.mean(y1 ** 2))
    assert scale > 0
    assert np.max(np.abs(y1 - y2)) <= 1e-10 * scale
    assert np.max(np.abs(y1 - y3)) <= 1e-10 * scale


def test_single_expert_is_a_dense_swiglu_mlp():
    shape = moe_synth.MoEShape("e1", E=1, k=1, H=128, I=64, renormalize=True, sigma=0.1)
    stack = _stack(shape, 3)
    x = moe_synth.activations(5, shape.H, 3).float().numpy()
    lg = moe_synth.logits(shape, 5, 3).numpy()
    y = oracle.moe_layer(x, lg, stack, 1)
    Wgu = torch.from_numpy(stack.gate_up(0))
    Wd = torch.from_numpy(stack.down(0))
    X = torch.from_numpy(x).double()
    g = X @ Wgu[:64].T
    u = X @ Wgu[64:].T
    ref = (torch.nn.functional.silu(g) * u) @ Wd.T
    assert np.allclose(y, ref.numpy(), rtol=1e-12, atol=1e-14)


def test_swiglu_closed_forms():
    gu = np.array([[0.0, 5.0, 2.0, 3.0], [40.0, -40.0, 1.0, 1.0]])
    h = oracle.swiglu(gu)
    assert h[0, 0] == 0.0
    assert abs(h[0, 1] - 5.0 / (1 + np.exp(-5.0)) * 3.0) < 1e-15
    assert abs(h[1, 0] - 40.0) < 1e-12       # silu(g) -> g for large g
    assert abs(h[1, 1]) < 1e-15              # silu(g) -> 0 for very negative g


def test_combine_one_hot_and_order():
    Yp = np.arange(12, dtype=np.float64).reshape(4, 3)
    inv_perm = np.array([2, 0, 3, 1])
    w = np.array([[1.0, 0.0], [0.25, 0.75]])
    Y = oracle.unpermute_combine(Yp, inv_perm, w)
    assert np.array_equal(Y[0], Yp[2])
    assert np.allclose(Y[1], 0.25 * Yp[3] + 0.75 * Yp[1])


def _tiny_setup():
    shape = moe_synth.TINY
    stack = _stack(shape, 0)
    x = moe_synth.activations(16, shape.H, 0).float().numpy()
    lg = moe_synth.logits(shape, 16, 0).numpy()
    ref = oracle.moe_layer(x, lg, stack, shape.k, shape.renormalize)
    return shape, stack, x, lg, ref


def _fails_tolerance(y, ref):
    rms = np.sqrt(np.mean(ref ** 2))
    rel = np.max(np.abs(y - ref) / np.maximum(np.abs(ref), rms))
    mae = np.mean(np.abs(y - ref))
    return rel > 1e-2 or mae > 1e-3 * rms


def test_transposed_input_weights_fail():
    # Planted mistake: reading each gate_up expert as [H, 2I] (the other
    # orientation) must not pass the layer's tolerance.
    shape, stack, x, lg, ref = _tiny_setup()
    H, I = shape.H, shape.I
    W = moe_synth.weights(shape, "gate_up", 0).numpy()
    Wt = np.ascontiguousarray(W.reshape(shape.E, H, 2 * I).transpose(0, 2, 1))
    p, a = oracle.quantize_blockwise(Wt)
    bad = oracle.ExpertStack(p, a.reshape(shape.E, -1), stack.packed_d, stack.absmax_d)
    y = oracle.moe_layer(x, lg, bad, shape.k, shape.renormalize)
    assert _fails_tolerance(y, ref)


def test_swapped_gate_and_up_fail():
    shape, stack, x, lg, ref = _tiny_setup()
    I = shape.I
    swapped = np.concatenate([stack.packed_gu[:, I:], stack.packed_gu[:, :I]], axis=1)
    a = stack.absmax_gu.reshape(shape.E, 2 * I, -1)
    a_sw = np.concatenate([a[:, I:], a[:, :I]], axis=1).reshape(shape.E, -1)
    bad = oracle.ExpertStack(swapped, a_sw, stack.packed_d, stack.absmax_d)
    y = oracle.moe_layer(x, lg, bad, shape.k, shape.renormalize)
    assert _fails_tolerance(y, ref)


def test_dropped_combine_weight_fails():
    shape, stack, x, lg, ref = _tiny_setup()
    idx, w = oracle.route_topk(lg, shape.k, shape.renormalize)
    offsets, rows, inv = oracle.permute_by_expert(idx, shape.E)
    GU = oracle.grouped_gemm(x, stack.packed_gu, stack.absmax_gu, offsets, gather=rows, k=shape.k)
    Yp = oracle.grouped_gemm(oracle.swiglu(GU), stack.packed_d, stack.absmax_d, offsets)
    w_bad = w.copy()
    w_bad[3, 1] = 0.0
    assert _fails_tolerance(oracle.unpermute_combine(Yp, inv, w_bad), ref)
    assert not _fails_tolerance(oracle.unpermute_combine(Yp, inv, w), ref)


def test_grouped_gemm_row_subset():
    shape, stack, x, lg, _ = _tiny_setup()
    idx, _ = oracle.route_topk(lg, shape.k)
    offsets, rows, _ = oracle.permute_by_expert(idx, shape.E)
    full = oracle.grouped_gemm(x, stack.packed_gu, stack.absmax_gu, offsets, gather=rows, k=shape.k)
    sub = oracle.grouped_gemm(x, stack.packed_gu, stack.absmax_gu, offsets, gather=rows,
                              k=shape.k, rows=[5, 0, 31])
    assert np.array_equal(sub, full[[5, 0, 31]])


def test_zipf_generator_structure():
    shape = moe_synth.QWEN3_30B
    lg = moe_synth.logits(shape, 4096, 0).numpy()
    idx, _ = oracle.route_topk(lg, shape.k)
    counts = np.bincount(idx.reshape(-1), minlength=shape.E)
    assert 1000 <= counts.max() <= 2000
    assert (counts == 0).sum() >= 1
