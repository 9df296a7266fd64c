"""Per-expert LoRA deltas over the frozen 4-bit expert weights, from the definition.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What the pages fix: per-expert LoRA / QLoRA adapters train over the frozen
4-bit base ("Jordan Anderson", jordananderson.work, section "4-bit
Mixture-of-Experts fine-tuning on small GPUs"; "MoE Training on Consumer
GPUs", cerinamroth.com/ml).  The readings taken here are the LoRA paper's
(Hu et al., 2021) usual form:

* expert e has adapters ``A_e [r, K]`` and ``B_e [N, r]`` for a weight
  ``W_e [N, K]`` (gate_up or down), and a common scale (alpha / r);
* the adapted product is ``W_e x + scale * B_e (A_e x)``; the delta is added to
  the projection's pre-activation, so for gate_up it comes before SiLU(gate)*up;
* a routed row p of expert e gets ``delta[p] = scale * B_e @ (A_e @ x_p)``.
"""

from __future__ import annotations

import numpy as np


def lora_delta(X: np.ndarray, expert_offsets: np.ndarray, lora_A: np.ndarray,
               lora_B: np.ndarray, scale: float, rows=None) -> np.ndarray:
    """``delta[p] = scale * B[e(p)] @ (A[e(p)] @ X[p])`` in fp64.

    ``X [M_total, K]`` (rows in expert-segment order), ``lora_A [E, r, K]``,
    ``lora_B [E, N, r]``; e(p) is the expert whose segment
    [offsets[e], offsets[e+1]) holds p.  Result ``[len(rows) or M_total, N]``."""
    X = np.asarray(X, dtype=np.float64)
    A = np.asarray(lora_A, dtype=np.float64)
    B = np.asarray(lora_B, dtype=np.float64)
    offsets = np.asarray(expert_offsets, dtype=np.int64)
    positions = np.arange(int(offsets[-1])) if rows is None else np.asarray(rows)
    experts = np.searchsorted(offsets, positions, side="right") - 1
    out = np.zeros((positions.size, B.shape[1]), dtype=np.float64)
    for i, p in enumerate(positions):
        e = int(experts[i])
        out[i] = float(scale) * (B[e] @ (A[e] @ X[p]))
    return out
