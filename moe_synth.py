"""Seeded synthetic inputs for the NF4 MoE layer (tests and bench).

This module only draws random numbers with the shapes, distributions and
structure of the workloads; it holds none of the layer's arithmetic (no
quantization, routing, GEMM or combine).  Both the CPU oracle's tests and the
GPU path's tests and bench take their inputs from here.

Workload shapes (the mixture-of-experts models the pages discuss):

* Tiny: E=8, top-2, hidden 256, expert intermediate 512, 16 tokens.
* OLMoE-shaped decode: E=64, top-8, hidden 2048, intermediate 1024, plain
  softmax (no renormalisation), token batches 1/4/16/64, N(0,1) logits.
* Qwen3-30B-A3B-shaped: E=128, top-8 renormalised, hidden 2048,
  intermediate 768; decode batches 1..64 and a 4096-token prefill, with
  Zipf-skewed routing (s = 1.1).
* Qwen3-235B-A22B-shaped: E=128, top-8 renormalised, hidden 4096,
  intermediate 1536, weights N(0, 0.015) with 0.1 % outliers at 8 sigma;
  uniform (N(0,1) logits) and Zipf-skewed routing.

Weights are fp32 N(0, sigma); activations bf16 N(0, 1); logits fp32.
"""

from __future__ import annotations

import dataclasses
import math

import torch

# Seed offsets so every tensor of a layer has its own stream.
_X, _LOGITS, _WGU, _WD, _OUTLIER, _LORA = 1, 2, 3, 4, 5, 6


@dataclasses.dataclass(frozen=True)
class MoEShape:
    name: str
    E: int
    k: int
    H: int
    I: int
    renormalize: bool
    sigma: float = 0.02
    routing: str = "normal"        # "normal" | "zipf"
    outlier_frac: float = 0.0
    zipf_s: float = 1.1
    zipf_beta: float = 0.3         # scale of log p_rank in the logits
    zipf_empty: int = 4            # lowest-ranked experts never chosen

    @property
    def nf4_bytes_per_expert(self) -> int:
        """Packed codes + fp32 absmax for gate_up [2I, H] and down [H, I]."""
        n = 3 * self.H * self.I
        return n // 2 + (n // 64) * 4


TINY = MoEShape("tiny", E=8, k=2, H=256, I=512, renormalize=True)
OLMOE = MoEShape("olmoe", E=64, k=8, H=2048, I=1024, renormalize=False)
QWEN3_30B = MoEShape("qwen3-30b-a3b", E=128, k=8, H=2048, I=768,
                     renormalize=True, routing="zipf")
QWEN3_235B = MoEShape("qwen3-235b-a22b", E=128, k=8, H=4096, I=1536,
                      renormalize=True, sigma=0.015, outlier_frac=1e-3)
# The same layer with Zipf-skewed routing (same weights for the same seed:
# the weights depend only on E, H, I, sigma and the outliers).
QWEN3_235B_ZIPF = dataclasses.replace(QWEN3_235B, name="qwen3-235b-a22b-zipf", routing="zipf")

SHAPES = {s.name: s for s in (TINY, OLMOE, QWEN3_30B, QWEN3_235B, QWEN3_235B_ZIPF)}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weights(shape: MoEShape, which: str, seed: int, experts=None,
            device="cpu") -> torch.Tensor:
    """fp32 expert weights, ``which`` in {"gate_up", "down"}.

    gate_up is ``[E, 2I, H]`` (rows [0, I) gate, [I, 2I) up), down is
    ``[E, H, I]``.  ``experts`` (a range or list) draws only those experts;
    every expert has its own generator, so a subset matches the full draw.
    """
    E = shape.E
    N, K = (2 * shape.I, shape.H) if which == "gate_up" else (shape.H, shape.I)
    off = _WGU if which == "gate_up" else _WD
    ids = list(range(E)) if experts is None else list(experts)
    out = torch.empty((len(ids), N, K), dtype=torch.float32, device=device)
    for i, e in enumerate(ids):
        g = _gen(seed * 1_000_003 + off * 10_007 + e, device)
        w = torch.randn((N, K), generator=g, device=device,
                        dtype=torch.float32) * shape.sigma
        if shape.outlier_frac > 0:
            go = _gen(seed * 1_000_003 + _OUTLIER * 10_007 + e + 7 * off, device)
            n_out = max(1, int(round(shape.outlier_frac * N * K)))
            pos = torch.randint(0, N * K, (n_out,), generator=go, device=device)
            sgn = torch.randint(0, 2, (n_out,), generator=go, device=device)
            val = (sgn.to(torch.float32) * 2 - 1) * (8.0 * shape.sigma)
            w.view(-1)[pos] = val
        out[i] = w
    return out


def activations(T: int, H: int, seed: int, device="cpu") -> torch.Tensor:
    """bf16 ``[T, H]`` ~ N(0, 1)."""
    g = _gen(seed * 1_000_003 + _X, device)
    return torch.randn((T, H), generator=g, device=device,
                       dtype=torch.float32).to(torch.bfloat16)


def logits(shape: MoEShape, T: int, seed: int, device="cpu") -> torch.Tensor:
    """fp32 router logits ``[T, E]``.

    "normal": i.i.d. N(0, 1) -- routing uniform in distribution.
    "zipf":  expert popularity p_r ~ r^-s over ranks r = 1..E, ranks assigned
    to experts by a seeded permutation; logits = beta * ln p_rank + N(0, 1),
    and the ``zipf_empty`` lowest-ranked experts get -1e4 so that empty
    experts always occur.  beta = 0.3 gives 0 to ~1500 rows per expert at
    4096 tokens x top-8 over 128 experts.
    """
    E = shape.E
    g = _gen(seed * 1_000_003 + _LOGITS, "cpu")
    if shape.routing == "normal":
        z = torch.randn((T, E), generator=g, dtype=torch.float32)
        return z.to(device)
    perm = torch.randperm(E, generator=g)
    ranks = torch.empty(E, dtype=torch.long)
    ranks[perm] = torch.arange(1, E + 1)
    logp = -shape.zipf_s * torch.log(ranks.to(torch.float64))
    logp = logp - torch.logsumexp(logp, 0)
    z = torch.randn((T, E), generator=g, dtype=torch.float32)
    out = (shape.zipf_beta * logp).to(torch.float32)[None, :] + z
    if shape.zipf_empty:
        out[:, ranks > E - shape.zipf_empty] = -1e4
    return out.to(device)


def lora_adapters(shape: MoEShape, which: str, rank: int, seed: int,
                  device="cpu"):
    """fp16 per-expert LoRA adapters for ``which`` in {"gate_up", "down"}:
    ``A [E, r, K] ~ N(0, 1/K)`` and ``B [E, N, r] ~ N(0, 0.02^2)`` (a trained
    B is small; LoRA starts it at zero)."""
    N, K = (2 * shape.I, shape.H) if which == "gate_up" else (shape.H, shape.I)
    off = _WGU if which == "gate_up" else _WD
    g = _gen(seed * 1_000_003 + _LORA * 10_007 + off, device)
    A = torch.randn((shape.E, rank, K), generator=g, device=device) / math.sqrt(K)
    B = torch.randn((shape.E, N, rank), generator=g, device=device) * 0.02
    return A.to(torch.float16), B.to(torch.float16)


def expected_distinct_experts(E: int, k: int, T: int) -> float:
    """E * (1 - (1 - k/E)^T): distinct experts hit under uniform routing."""
    return E * (1.0 - math.pow(1.0 - k / E, T))
