"""Backward of the 4-bit mixture-of-experts layer with frozen experts, by the chain rule.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What the pages fix: the kernel is differentiable, fine-tuning computes on the
packed 4-bit weights instead of unpacking them, the frozen 4-bit stack stays
byte-identical, and the backward is one launch ("grouped-nf4-gemm &
experts-4bit", jordananderson-pages.pages.dev, fourth bullet).  They print no
formulas.  The readings taken here are the chain rule through the forward
layer of ``oracle.moe``:

* differentiated inputs: the activations x and the router logits (and, with
  adapters, the LoRA matrices); the 4-bit weights are constants, so no weight
  gradient exists;
* which experts are chosen is piecewise constant in the logits: no gradient
  flows through the selection, only through the weights w[t, j];
* the transposed grouped GEMM is ``out[p] = W[e(p)]^T g[p]`` on the same
  dequantized values the forward multiplies by;
* SwiGLU: with s = sigmoid(g), silu(g) = g s and silu'(g) = s (1 + g (1 - s));
  dg = dh * u * silu'(g), du = dh * silu(g);
* combine: dYp[pos(t, j)] = w[t, j] dY[t] and dw[t, j] = <dY[t], Yp[pos(t, j)]>;
* routing: without renormalisation w_j = p_{e_j} (softmax over all E), so
  dl_i = sum_j dw_j p_{e_j} (delta_{i e_j} - p_i); with it w is the softmax
  over the k selected logits, so dl_{e_j} = w_j (dw_j - sum_j' dw_j' w_j') and
  the other logits get 0;
* the gather of token rows into routed rows has the scatter-add as adjoint:
  dx[t] sums the input gradients of its k routed rows;
* LoRA (``oracle.lora``): delta = scale B (A x), so dx = scale A^T (B^T g),
  dB = scale sum_p g (A x_p)^T and dA = scale sum_p (B^T g) x_p^T per expert.
"""

from __future__ import annotations

import numpy as np

from .moe import ExpertStack, _silu, grouped_gemm, swiglu, unpermute_combine
from .nf4 import dequantize_blockwise
from .routing import permute_by_expert, route_topk


def _sigmoid(g: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-g))


def grouped_gemm_t(G: np.ndarray, packed: np.ndarray, absmax: np.ndarray,
                   expert_offsets: np.ndarray) -> np.ndarray:
    """Transposed grouped NF4 GEMM: ``out[p] = W[e(p)]^T @ G[p]``.

    ``G [M_total, N]``, ``packed uint8[E, N, K/2]``, ``absmax float32[E, N*K/64]``;
    fp64 result ``[M_total, K]``.  The weights are those of ``grouped_gemm``."""
    G = np.asarray(G, dtype=np.float64)
    E, N, half_k = packed.shape
    offsets = np.asarray(expert_offsets, dtype=np.int64)
    out = np.zeros((int(offsets[-1]), 2 * half_k), dtype=np.float64)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi > lo:
            W = dequantize_blockwise(packed[e], absmax[e].reshape(N, -1))
            for p in range(lo, hi):
                out[p] = W.T @ G[p]
    return out


def swiglu_backward(gu: np.ndarray, dh: np.ndarray) -> np.ndarray:
    """``gu [M, 2I]`` (gate | up pre-activations), ``dh [M, I]`` -> ``d_gu [M, 2I]``."""
    gu = np.asarray(gu, dtype=np.float64)
    dh = np.asarray(dh, dtype=np.float64)
    I = gu.shape[1] // 2
    g, u = gu[:, :I], gu[:, I:]
    s = _sigmoid(g)
    dsilu = s * (1.0 + g * (1.0 - s))
    return np.concatenate([dh * u * dsilu, dh * g * s], axis=1)


def combine_backward(dY: np.ndarray, Yp: np.ndarray, inv_perm: np.ndarray,
                     weights: np.ndarray):
    """Adjoint of ``unpermute_combine``: ``(dYp [T*k, H], dw [T, k])``."""
    dY = np.asarray(dY, dtype=np.float64)
    Yp = np.asarray(Yp, dtype=np.float64)
    weights = np.asarray(weights, dtype=np.float64)
    T, k = weights.shape
    dYp = np.zeros_like(Yp)
    dw = np.zeros((T, k), dtype=np.float64)
    for t in range(T):
        for j in range(k):
            pos = int(inv_perm[t * k + j])
            dYp[pos] = weights[t, j] * dY[t]
            dw[t, j] = dY[t] @ Yp[pos]
    return dYp, dw


def route_backward(logits: np.ndarray, idx: np.ndarray, dw: np.ndarray,
                   renormalize: bool = True) -> np.ndarray:
    """Gradient of the routing weights' loss w.r.t. the logits, ``[T, E]``.

    ``idx [T, k]`` is the selection ``route_topk`` made (held fixed);
    ``dw [T, k]`` the gradient w.r.t. its weights."""
    l64 = np.asarray(logits, dtype=np.float64)
    dw = np.asarray(dw, dtype=np.float64)
    T, E = l64.shape
    out = np.zeros((T, E), dtype=np.float64)
    for t in range(T):
        sel = [int(e) for e in idx[t]]
        if renormalize:
            z = l64[t, sel] - l64[t, sel].max()
            w = np.exp(z) / np.exp(z).sum()
            c = float(dw[t] @ w)
            for j, e in enumerate(sel):
                out[t, e] += w[j] * (dw[t, j] - c)
        else:
            z = l64[t] - l64[t].max()
            p = np.exp(z) / np.exp(z).sum()
            for j, e in enumerate(sel):
                out[t] -= dw[t, j] * p[e] * p
                out[t, e] += dw[t, j] * p[e]
    return out


def moe_layer_backward(x: np.ndarray, logits: np.ndarray, stack: ExpertStack, k: int,
                       renormalize: bool, dY: np.ndarray, with_dw: bool = False):
    """``(dx [T, H], dlogits [T, E])`` of ``oracle.moe_layer`` for the output
    gradient ``dY [T, H]``, one token and one routed expert at a time.
    ``with_dw``: also return ``(idx [T, k], dw [T, k])``, the selection and
    the gradient w.r.t. its routing weights."""
    x = np.asarray(x, dtype=np.float64)
    dY = np.asarray(dY, dtype=np.float64)
    idx, w = route_topk(np.asarray(logits, dtype=np.float32), k, renormalize)
    T = x.shape[0]
    I = stack.I
    dx = np.zeros_like(x)
    dw = np.zeros((T, k), dtype=np.float64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            Wgu, Wd = stack.gate_up(e), stack.down(e)
            gu = Wgu @ x[t]
            h = _silu(gu[:I]) * gu[I:]
            dw[t, j] = dY[t] @ (Wd @ h)
            dh = Wd.T @ (w[t, j] * dY[t])
            dgu = swiglu_backward(gu[None], dh[None])[0]
            dx[t] += Wgu.T @ dgu
    dl = route_backward(logits, idx, dw, renormalize)
    return (dx, dl, idx, dw) if with_dw else (dx, dl)


def moe_layer_backward_permuted(x, logits, stack: ExpertStack, k: int, renormalize: bool,
                                dY):
    """The same gradients through the grouped steps a one-launch backward runs:
    recompute the forward's routed rows, then combine backward, transposed
    grouped down, SwiGLU backward, transposed grouped gate_up, scatter-add."""
    x = np.asarray(x, dtype=np.float64)
    idx, w = route_topk(np.asarray(logits, dtype=np.float32), k, renormalize)
    offsets, sorted_rows, inv_perm = permute_by_expert(idx, stack.E)
    GU = grouped_gemm(x, stack.packed_gu, stack.absmax_gu, offsets, gather=sorted_rows, k=k)
    Yp = grouped_gemm(swiglu(GU), stack.packed_d, stack.absmax_d, offsets)
    dYp, dw = combine_backward(dY, Yp, inv_perm, w)
    dH = grouped_gemm_t(dYp, stack.packed_d, stack.absmax_d, offsets)
    dXp = grouped_gemm_t(swiglu_backward(GU, dH), stack.packed_gu, stack.absmax_gu, offsets)
    dx = np.zeros_like(x)
    for p, f in enumerate(sorted_rows):
        dx[int(f) // k] += dXp[p]
    return dx, route_backward(logits, idx, dw, renormalize)


def lora_backward(X: np.ndarray, expert_offsets: np.ndarray, lora_A: np.ndarray,
                  lora_B: np.ndarray, scale: float, G: np.ndarray):
    """Gradients of ``<G, lora_delta(X, ...)>``: ``(dX [M, K], dA [E, r, K],
    dB [E, N, r])``."""
    X = np.asarray(X, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    A = np.asarray(lora_A, dtype=np.float64)
    B = np.asarray(lora_B, dtype=np.float64)
    offsets = np.asarray(expert_offsets, dtype=np.int64)
    dX = np.zeros_like(X[: int(offsets[-1])])
    dA = np.zeros_like(A)
    dB = np.zeros_like(B)
    for e in range(A.shape[0]):
        for p in range(int(offsets[e]), int(offsets[e + 1])):
            u = A[e] @ X[p]
            v = B[e].T @ G[p]
            dX[p] = scale * (A[e].T @ v)
            dB[e] += scale * np.outer(G[p], u)
            dA[e] += scale * np.outer(v, X[p])
    return dX, dA, dB
