"""Top-k softmax routing and the token->expert permutation, from definitions.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The pages name a router ("real attention and router", "grouped-nf4-gemm &
experts-4bit", jordananderson-pages.pages.dev, second bullet) and a kernel
that covers all active experts in one launch (same section, first bullet),
which needs each expert's routed rows as one contiguous segment.  They give
no formula; the readings taken here are:

* selection on the fp32 logits: the k largest, in descending order, equal
  logits resolved towards the lower expert index;
* weights: softmax over all E logits, then, with ``renormalize``, divided by
  their sum over the k selected experts (equivalently a softmax over the k
  selected logits); without it, the plain softmax probabilities;
* permutation: routed rows are the flat ids f = t*k + j; they are ordered
  stably by expert, then by f.  ``expert_offsets[e]`` is the first position
  of expert e's segment, ``expert_offsets[E] == T*k``; ``sorted_rows[p]`` is
  the flat id at position p and ``inv_perm[f]`` the position of flat id f.
"""

from __future__ import annotations

import numpy as np


def route_topk(logits: np.ndarray, k: int, renormalize: bool = True):
    """``logits float32[T, E]`` -> ``(idx int32[T, k], weights float64[T, k])``."""
    logits = np.asarray(logits)
    if logits.dtype != np.float32:
        raise TypeError("route_topk expects float32 logits")
    T, E = logits.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    if not np.all(np.isfinite(logits)):
        raise ValueError("non-finite logits are outside the router's contract")
    # Stable sort of the negated logits: descending, ties keep the lower index.
    order = np.argsort(-logits, axis=1, kind="stable")
    idx = order[:, :k].astype(np.int32)

    l64 = logits.astype(np.float64)
    m = l64.max(axis=1, keepdims=True)
    ex = np.exp(l64 - m)
    p = ex / ex.sum(axis=1, keepdims=True)
    w = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    if renormalize:
        w = w / w.sum(axis=1, keepdims=True)
    return idx, w


def permute_by_expert(idx: np.ndarray, E: int):
    """Stable counting sort of routed rows by expert.

    ``idx int32[T, k]`` -> ``(expert_offsets int32[E+1], sorted_rows int32[T*k],
    inv_perm int32[T*k])``.
    """
    flat = np.asarray(idx, dtype=np.int64).reshape(-1)
    if flat.size and (flat.min() < 0 or flat.max() >= E):
        raise ValueError("expert index out of range")
    counts = np.bincount(flat, minlength=E)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    sorted_rows = np.argsort(flat, kind="stable")
    inv_perm = np.empty_like(sorted_rows)
    inv_perm[sorted_rows] = np.arange(flat.size)
    return (offsets.astype(np.int32), sorted_rows.astype(np.int32),
            inv_perm.astype(np.int32))
