#!/usr/bin/env python
"""Benchmark of the NF4 grouped mixture-of-experts layer on B200.

One step = one pass of the whole hot path -- route + permute, grouped gate_up
GEMM with fused SwiGLU, grouped down GEMM, combine -- over one token batch,
through a stack of independent MoE layers whose NF4 weights together exceed
the 126 MB L2 (every layer's weights stream from HBM once per step).

Headline workload (the N = 1 line's ``value``): the largest single-GPU shape,
a Qwen3-235B-A22B-shaped layer (E=128, top-8, hidden 4096, expert
intermediate 1536, 1.36 GB of NF4) at a 2048-token prefill, where both grouped
GEMMs run on the tensor cores.  Every other configuration of the workload list
-- Tiny, OLMoE decode T = 1/4/16/64, Qwen3-30B-A3B decode (48 layers) and
prefill, Qwen3-235B decode T = 1/8/32 and the Zipf-routed prefill -- is timed
in the same run and reported under ``workloads``, each with its own roofline
and CPU-oracle baseline.  ``--config`` / ``--tokens`` time one workload alone.

Prints ONE JSON line (rank 0).  ``--impl reference`` times the CPU oracle
instead (bounded samples of the same workload).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import moe_synth  # noqa: E402

CONFIGS = {
    # name: (shape, T, layers)
    "olmoe-decode": (moe_synth.OLMOE, 64, 16),
    "qwen3-30b-decode": (moe_synth.QWEN3_30B, 64, 48),
    "qwen3-30b-prefill": (moe_synth.QWEN3_30B, 4096, 2),
    "qwen3-235b-decode": (moe_synth.QWEN3_235B, 32, 8),
    "qwen3-235b-prefill": (moe_synth.QWEN3_235B, 2048, 1),
    "qwen3-235b-prefill-zipf": (moe_synth.QWEN3_235B_ZIPF, 2048, 1),
    "tiny": (moe_synth.TINY, 16, 128),
}
HEADLINE = "qwen3-235b-prefill"
# The rest of the workload list, timed after the headline: (config, T).
SWEEP = [("tiny", 16),
         ("olmoe-decode", 1), ("olmoe-decode", 4), ("olmoe-decode", 16), ("olmoe-decode", 64),
         ("qwen3-30b-decode", 1), ("qwen3-30b-decode", 8), ("qwen3-30b-decode", 64),
         ("qwen3-30b-prefill", 4096),
         ("qwen3-235b-decode", 1), ("qwen3-235b-decode", 8), ("qwen3-235b-decode", 32),
         ("qwen3-235b-prefill-zipf", 2048)]
SWEEP_STEPS = 20          # timed steps per sweep workload (at most --steps)
# Nominal B200 figures, for the second fraction each roofline carries.
NOMINAL_HBM_GBS, NOMINAL_BF16_TFLOPS = 8000.0, 2250.0


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--config", choices=sorted(CONFIGS), default=HEADLINE)
    p.add_argument("--no-sweep", action="store_true",
                   help="time the headline (or --config) workload only")
    p.add_argument("--tokens", type=int, default=None, help="token batch T")
    p.add_argument("--layers", type=int, default=None)
    p.add_argument("--algo", choices=["auto", "gemv", "tc", "tc_pair"], default="auto")
    p.add_argument("--weights", choices=["nf4", "int4", "mxfp4"], default="nf4",
                   help="expert weight format (int4: grouped GPTQ-style codes; mxfp4: e2m1 + "
                        "e8m0 per 32)")
    p.add_argument("--backward", action="store_true",
                   help="time forward + backward of each layer (4-bit experts frozen)")
    p.add_argument("--lora", type=int, default=0, metavar="RANK",
                   help="per-expert LoRA adapters of this rank on both projections "
                        "(0 = none)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--seed", type=int, default=0)
    return p.parse_args()


# ----------------------------------------------------------------- utilities

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def recorded_traffic(kernel_source, workload):
    """DRAM bytes per launch from profiles/kernel_traffic.txt, or None when the
    kernel source changed since the capture (sha256 mismatch) or no capture
    of this workload exists."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "kernel_traffic.txt")
    src = os.path.join(ROOT, "bit_mixture_experts_route_b200", "csrc", kernel_source)
    if not (os.path.exists(path) and os.path.exists(src)):
        return None
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) == 4 and not line.startswith("#") and parts[0] == kernel_source \
                    and parts[1] == sha and parts[2] == workload:
                return float(parts[3])
    return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons every 20 ms.  Each sample carries
    nvidia-smi's own timestamp; only samples taken between mark_start() and
    mark_end() (the timed region) enter the summary."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.6)  # nvidia-smi's start-up, before the timed region
        except OSError:
            self.proc = None
        return self

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    @staticmethod
    def _stamp(text):
        import datetime
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(text, fmt).timestamp()
            except ValueError:
                continue
        return None

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        outside = 0
        for ln in getattr(self, "lines", []):
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 10:
                continue
            ts = self._stamp(parts[0])
            if self.t0 is not None and ts is not None and not (
                    self.t0 - 0.02 <= ts <= (self.t1 or ts) + 0.02):
                outside += 1
                continue
            try:
                sm.append(float(parts[2]))
                smax = float(parts[3])
            except ValueError:
                continue
            for nm, val in zip(names, parts[6:10]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "samples_outside_timed_region": outside}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm),
                "samples_outside_timed_region": outside}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """Max of a host float over all ranks (on the process group's device)."""
    if world <= 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(seed, rank):
    """Each replica draws its own token batch and weights (weak scaling)."""
    return seed + 7919 * rank


# ----------------------------------------------------------------- workload

# bytes per weight: the 4-bit code plus its share of the scales (NF4: fp32
# absmax per 64; INT4: fp16 scale + zero in 4 B per 128; MXFP4: 1 B per 32)
BYTES_PER_WEIGHT = {"nf4": 0.5625, "int4": 0.53125, "mxfp4": 0.53125}
DECODE_KERNEL_SOURCE = {"nf4": "grouped_gemm_decode.cu", "int4": "grouped_gemm_decode.cu",
                        "mxfp4": "grouped_gemm_decode.cu"}

class Workload:
    """One configuration's NF4 (or INT4, MXFP4) layer stacks on the device,
    and the token-batch buffers of the current ``T`` (``set_tokens``)."""

    def __init__(self, shape, T, layers, seed, device="cuda", weights="nf4", lora=0,
                 backward=False):
        import bit_mixture_experts_route_b200 as moe
        self.moe = moe
        self.shape, self.L, self.seed, self.dev = shape, layers, seed, device
        self.fmt = weights
        self.lora = lora
        self.backward = backward
        quantize = {"nf4": moe.nf4_quantize, "int4": moe.int4_quantize,
                    "mxfp4": moe.mxfp4_quantize}[weights]
        self.stacks = []
        for layer in range(layers):
            s = seed * 1000 + layer
            w = moe_synth.weights(shape, "gate_up", s, device=device)
            p_gu, a_gu = quantize(w)
            del w
            w = moe_synth.weights(shape, "down", s, device=device)
            p_d, a_d = quantize(w)
            del w
            self.stacks.append((p_gu, a_gu, p_d, a_d))
        torch.cuda.empty_cache()
        if lora:
            self.adapters = [moe_synth.lora_adapters(shape, "gate_up", lora, seed * 1000 + layer,
                                                     device=device)
                             + moe_synth.lora_adapters(shape, "down", lora, seed * 1000 + layer,
                                                       device=device)
                             for layer in range(layers)]
        self.set_tokens(T)

    def set_tokens(self, T):
        """Inputs and intermediates of a T-token batch (``shape`` may differ
        from the weights' in its routing only)."""
        moe, shape, seed, dev = self.moe, self.shape, self.seed, self.dev
        self.T = T
        self.X = moe_synth.activations(T, shape.H, seed, device=dev)
        self.logits = torch.stack([moe_synth.logits(shape, T, seed * 1000 + layer, device=dev)
                                   for layer in range(self.L)])
        k, E, H, I = shape.k, shape.E, shape.H, shape.I
        M = T * k
        self.route = {
            "topk_idx": torch.empty((T, k), dtype=torch.int32, device=dev),
            "topk_w": torch.empty((T, k), dtype=torch.float32, device=dev),
            "expert_offsets": torch.empty((E + 1,), dtype=torch.int32, device=dev),
            "sorted_rows": torch.empty((M,), dtype=torch.int32, device=dev),
            "inv_perm": torch.empty((M,), dtype=torch.int32, device=dev),
        }
        self.rws = torch.empty((max(moe.route_permute_workspace_size(T, E, k), 256),),
                               dtype=torch.uint8, device=dev)
        self.Xp = torch.empty((M, H), dtype=torch.float16, device=dev)
        self.Hbuf = torch.empty((M, I), dtype=torch.float16, device=dev)
        self.Yp = torch.empty((M, H), dtype=torch.float16, device=dev)
        self.Y = torch.empty((T, H), dtype=torch.float32, device=dev)
        self.lws = torch.empty((max(moe.layer_workspace_size(T, E, k, H, I), 256),),
                               dtype=torch.uint8, device=dev)
        if self.lora or self.backward:
            # both GEMMs write fp32 pre-activations (the adapters add their
            # term in place; the backward needs gate_up's), SwiGLU standalone
            self.GU = torch.empty((M, 2 * I), dtype=torch.float32, device=dev)
            self.Yp32 = torch.empty((M, H), dtype=torch.float32, device=dev)
        if self.backward:
            g = torch.Generator(device=dev)
            g.manual_seed(seed * 1000 + 999)
            self.dY = torch.randn((T, H), generator=g, device=dev, dtype=torch.float32)
            self.ones = torch.ones((T, k), dtype=torch.float32, device=dev)
            self.dX = torch.empty((T, H), dtype=torch.float32, device=dev)

    def layer(self, layer, algo="auto", ev=None, X=None, logits=None):
        moe, sh, T = self.moe, self.shape, self.T
        X = self.X if X is None else X
        logits = self.logits[layer] if logits is None else logits
        p_gu, a_gu, p_d, a_d = self.stacks[layer]
        r = moe.route_permute(logits, sh.k, sh.renormalize, workspace=self.rws, out=self.route)
        M = T * sh.k
        moe.permute_rows(X, r["sorted_rows"], sh.k, out=self.Xp)
        if self.lora or self.backward:
            self._adapted_layer(layer, r, M, algo, ev, logits)
            return
        if ev is not None:
            ev[0].record()
        self._gemm(self.Xp, p_gu, a_gu, r["expert_offsets"], M, self.Hbuf, algo, "swiglu")
        if ev is not None:
            ev[1].record()
        self._gemm(self.Hbuf, p_d, a_d, r["expert_offsets"], M, self.Yp, algo)
        moe.unpermute_combine(self.Yp, r["inv_perm"], r["topk_w"], out=self.Y)

    def _gemm(self, A, packed, scales, offsets, M, out, algo, epilogue="none"):
        if self.fmt == "int4":
            self.moe.int4_grouped_gemm(A, packed, scales, offsets, M, epilogue=epilogue, out=out,
                                       algo=algo)
        elif self.fmt == "mxfp4":
            self.moe.mxfp4_grouped_gemm(A, packed, scales, offsets, M, epilogue=epilogue, out=out,
                                        algo=algo)
        else:
            self.moe.nf4_grouped_gemm(A, packed, scales, offsets, M, epilogue=epilogue, out=out,
                                      algo=algo)

    def _adapted_layer(self, layer, r, M, algo, ev, logits):
        """Forward with fp32 pre-activations (plus the adapters' deltas when
        adapted), then, with --backward, the layer's backward for a fixed
        output gradient: combine backward, transposed down, SwiGLU backward,
        transposed gate_up, scatter-add into tokens, routing backward."""
        moe = self.moe
        p_gu, a_gu, p_d, a_d = self.stacks[layer]
        off = r["expert_offsets"]
        if self.lora:
            A_gu, B_gu, A_d, B_d = self.adapters[layer]
            scale = 32.0 / self.lora     # alpha = 32
        if ev is not None:
            ev[0].record()
        self._gemm(self.Xp, p_gu, a_gu, off, M, self.GU, algo)
        if ev is not None:
            ev[1].record()
            ev[2].record()
        if self.lora:
            moe.lora_delta(self.Xp, off, A_gu, B_gu, scale, self.GU, M_total=M)
        if ev is not None:
            ev[3].record()
        moe.swiglu(self.GU, out=self.Hbuf)
        self._gemm(self.Hbuf, p_d, a_d, off, M, self.Yp32, algo)
        if self.lora:
            moe.lora_delta(self.Hbuf, off, A_d, B_d, scale, self.Yp32, M_total=M)
        moe.unpermute_combine(self.Yp32, r["inv_perm"], r["topk_w"], out=self.Y)
        if self.backward:
            sh = self.shape
            if self.tc_backward():
                # tensor cores: fp16 row gradients, the transposed down GEMM
                # and the SwiGLU backward in one launch, the transposed gate_up
                dYp, dw = moe.combine_backward(self.dY, self.Yp32, r["inv_perm"], r["topk_w"],
                                               dyp_dtype=torch.float16)
                dGU = moe.nf4_down_backward(dYp, p_d, a_d, off, M, self.GU,
                                            out_dtype=torch.float16)
                dXp = moe.nf4_grouped_gemm_t(dGU, p_gu, a_gu, off, M, algo="tc")
            else:
                dYp, dw = moe.combine_backward(self.dY, self.Yp32, r["inv_perm"], r["topk_w"])
                dH = moe.nf4_grouped_gemm_t(dYp, p_d, a_d, off, M, algo="gemv")
                dGU = moe.swiglu_backward(self.GU, dH)
                dXp = moe.nf4_grouped_gemm_t(dGU, p_gu, a_gu, off, M, algo="gemv")
            moe.unpermute_combine(dXp, r["inv_perm"], self.ones, out=self.dX)
            moe.route_backward(logits, r["topk_idx"], r["topk_w"], dw, sh.renormalize)

    def tc_backward(self):
        """The backward runs on the tensor cores from 36 routed rows per expert
        on average (the forward's rule) when the shapes allow it."""
        sh = self.shape
        return (self.T * sh.k >= 36 * sh.E and sh.H % 64 == 0 and sh.I % 256 == 0
                and sh.H % 256 == 0 and (2 * sh.I) % 64 == 0)

    def lora_bytes(self, d):
        """Algorithmic bytes of the gate_up adapter launch: the distinct
        experts' A and B, the routed input rows, the fp32 pre-activation read
        and written."""
        sh, M = self.shape, self.T * self.shape.k
        return (d * self.lora * (sh.H + 2 * sh.I) * 2 + M * sh.H * 2
                + 2 * M * 2 * sh.I * 4)

    def step(self, algo="auto", evs=None, fused=False):
        """One pass through every layer.  ``fused``: each layer is the one C
        call ``moe_layer_forward`` (its GEMMs in chain mode: each starts
        streaming its weights while the kernel before it finishes); else the
        exported calls one by one, with CUDA events around gate_up."""
        if fused and self.fmt == "nf4" and not (self.lora or self.backward) and algo == "auto":
            sh = self.shape
            for layer in range(self.L):
                self.moe.layer_forward(self.X, self.logits[layer], sh.k, sh.renormalize,
                                       *self.stacks[layer], workspace=self.lws, out=self.Y)
            return
        for layer in range(self.L):
            self.layer(layer, algo, None if evs is None else evs[layer])

    # Algorithmic work ----------------------------------------------------
    def distinct_experts(self):
        """Experts with >= 1 routed row, per layer (from expert_offsets)."""
        out = []
        for layer in range(self.L):
            r = self.moe.route_permute(self.logits[layer], self.shape.k, self.shape.renormalize)
            off = r["expert_offsets"].cpu().numpy()
            out.append(int(np.count_nonzero(np.diff(off))))
        return out

    def gate_up_bytes(self, d):
        sh, T = self.shape, self.T
        w = d * (2 * sh.I * sh.H) * BYTES_PER_WEIGHT[self.fmt]
        # output: fp16 SwiGLU rows, or fp32 gate_up pre-activations when adapted
        out = T * sh.k * 2 * sh.I * 4 if (self.lora or self.backward) else T * sh.k * sh.I * 2
        return w + T * sh.H * 2 + out

    def layer_bytes(self, d):
        sh, T = self.shape, self.T
        per_w = BYTES_PER_WEIGHT[self.fmt]
        return d * 3 * sh.H * sh.I * per_w + T * sh.H * 2 + T * sh.E * 4 + T * sh.H * 4

    def gate_up_flops(self):
        sh = self.shape
        return 2.0 * self.T * sh.k * sh.H * 2 * sh.I


# ----------------------------------------------------------------- CPU oracle

def oracle_sample(shape, T, seed, n_tokens, start_token=0, threads=None, weights="nf4"):
    """Time the oracle on ``n_tokens`` tokens of layer 0: dequantize the NF4
    (or INT4, MXFP4) experts they need and run the per-token expert MLPs.  Weights
    come from the same generator as the GPU run; quantization is untimed
    setup."""
    import oracle
    s = seed * 1000
    X = moe_synth.activations(T, shape.H, seed).float().numpy()
    lg = moe_synth.logits(shape, T, s).numpy()
    idx, _ = oracle.route_topk(lg, shape.k, shape.renormalize)
    toks = [(start_token + i) % T for i in range(n_tokens)]
    experts = sorted({int(e) for t in toks for e in idx[t]})
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    w_gu = moe_synth.weights(shape, "gate_up", s, experts=experts, device=dev).cpu().numpy()
    w_d = moe_synth.weights(shape, "down", s, experts=experts, device=dev).cpu().numpy()
    E, I, H = shape.E, shape.I, shape.H
    if weights == "mxfp4":
        p_gu = np.zeros((E, 2 * I, H // 2), np.uint8)
        s_gu = np.zeros((E, 2 * I, H // 32), np.uint8)
        p_d = np.zeros((E, H, I // 2), np.uint8)
        s_d = np.zeros((E, H, I // 32), np.uint8)
        for i, e in enumerate(experts):
            p_gu[e], s_gu[e] = oracle.quantize_mxfp4(w_gu[i])
            p_d[e], s_d[e] = oracle.quantize_mxfp4(w_d[i])
        stack = oracle.Mxfp4ExpertStack(p_gu, s_gu, p_d, s_d)
        t0 = time.perf_counter()
        oracle.moe_layer(X, lg, stack, shape.k, shape.renormalize, tokens=toks)
        return n_tokens, time.perf_counter() - t0
    if weights == "int4":
        p_gu = np.zeros((E, 2 * I, H // 2), np.uint8)
        m_gu = np.zeros((E, 2 * I, H // 128), np.uint32)
        p_d = np.zeros((E, H, I // 2), np.uint8)
        m_d = np.zeros((E, H, I // 128), np.uint32)
        for i, e in enumerate(experts):
            p_gu[e], m_gu[e] = oracle.quantize_int4_grouped(w_gu[i])
            p_d[e], m_d[e] = oracle.quantize_int4_grouped(w_d[i])
        stack = oracle.Int4ExpertStack(p_gu, m_gu, p_d, m_d)
        t0 = time.perf_counter()
        oracle.moe_layer(X, lg, stack, shape.k, shape.renormalize, tokens=toks)
        return n_tokens, time.perf_counter() - t0
    p_gu = np.zeros((E, 2 * I, H // 2), np.uint8)
    a_gu = np.zeros((E, 2 * I * H // 64), np.float32)
    p_d = np.zeros((E, H, I // 2), np.uint8)
    a_d = np.zeros((E, H * I // 64), np.float32)
    for i, e in enumerate(experts):
        p, a = oracle.quantize_blockwise(w_gu[i])
        p_gu[e], a_gu[e] = p, a.reshape(-1)
        p, a = oracle.quantize_blockwise(w_d[i])
        p_d[e], a_d[e] = p, a.reshape(-1)
    stack = oracle.ExpertStack(p_gu, a_gu, p_d, a_d)
    t0 = time.perf_counter()
    oracle.moe_layer(X, lg, stack, shape.k, shape.renormalize, tokens=toks)
    dt = time.perf_counter() - t0
    return n_tokens, dt


def cpu_cores():
    try:
        aff = len(os.sched_getaffinity(0))
    except AttributeError:
        aff = os.cpu_count()
    threads = aff
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        if info:
            threads = max(int(d.get("num_threads", 1)) for d in info)
    except Exception:
        pass
    return os.cpu_count(), aff, threads


def run_reference(args, shape, T, layers):
    """The oracle as the reference arm: its per-token expert MLPs on a fixed
    sample of layer 0 (quantization and the one-time dequantization of the
    sample's experts are untimed set-up), K timed steps."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1 and rank != 0:
        return
    import oracle
    n_tok = 2
    s = args.seed * 1000
    X = moe_synth.activations(T, shape.H, args.seed).float().numpy()
    lg = moe_synth.logits(shape, T, s).numpy()
    idx, _ = oracle.route_topk(lg, shape.k, shape.renormalize)
    toks = list(range(n_tok))
    experts = sorted({int(e) for t in toks for e in idx[t]})
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    w_gu = moe_synth.weights(shape, "gate_up", s, experts=experts, device=dev).cpu().numpy()
    w_d = moe_synth.weights(shape, "down", s, experts=experts, device=dev).cpu().numpy()
    E, I, H = shape.E, shape.I, shape.H
    p_gu = np.zeros((E, 2 * I, H // 2), np.uint8)
    a_gu = np.zeros((E, 2 * I * H // 64), np.float32)
    p_d = np.zeros((E, H, I // 2), np.uint8)
    a_d = np.zeros((E, H * I // 64), np.float32)
    for i, e in enumerate(experts):
        p, a = oracle.quantize_blockwise(w_gu[i])
        p_gu[e], a_gu[e] = p, a.reshape(-1)
        p, a = oracle.quantize_blockwise(w_d[i])
        p_d[e], a_d[e] = p, a.reshape(-1)
    stack = oracle.ExpertStack(p_gu, a_gu, p_d, a_d)
    for _ in range(max(1, args.warmup)):   # the first call dequantizes the experts
        oracle.moe_layer(X, lg, stack, shape.k, shape.renormalize, tokens=toks)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.moe_layer(X, lg, stack, shape.k, shape.renormalize, tokens=toks)
    total_t = time.perf_counter() - t0
    total_tok = n_tok * args.steps
    value = total_tok / total_t
    ncpu, aff, threads = cpu_cores()
    line = {
        "impl": "reference", "metric": "MoE layer tokens/s", "value": value,
        "unit": "tokens/s", "n_gpus": 0, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_t / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.config, "T": T, "layers": layers, "E": shape.E,
                   "k": shape.k, "hidden": shape.H, "intermediate": shape.I},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"the same {n_tok} tokens of layer 0 each step (their {len(experts)} "
                                   f"experts quantized and dequantized once, untimed); host "
                                   f"cpu_count={ncpu}, affinity={aff}"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- one workload

def _cuda_fault(exc):
    """An exception that reports a fault on the device (the context is lost)
    rather than a call that stream capture does not allow."""
    msg = str(exc)
    return any(m in msg for m in ("launch failure", "illegal", "misaligned", "Xid",
                                   "device-side assert", "unspecified"))


def graphed_replay(wl, algo, steps, warmup, world, local):
    """The layer steps captured as one CUDA graph and replayed ``steps``
    times (how a decode server issues a step): same kernels and work as the
    eager launches, no per-launch host cost.  Returns (timing dict or error,
    clock summary)."""
    stream = torch.cuda.current_stream()
    g = None
    try:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            wl.step(algo, fused=True)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            wl.step(algo, fused=True)
        for _ in range(max(3, warmup)):
            g.replay()
        torch.cuda.synchronize()
        captured = 1.0
    except Exception as exc:  # noqa: BLE001
        if _cuda_fault(exc):
            raise  # a fault on the device is not a capture failure
        err = {"error": str(exc)[:200]}
        captured = 0.0
    # every rank takes the same collective steps: time only if all captured
    if -max_over_ranks(-captured, world) <= 0:
        del g
        return (err if captured == 0.0 else {"error": "another rank failed to capture"}), None
    gs, ge = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        clk.mark_start()
        gs.record()
        for _ in range(steps):
            g.replay()
        ge.record()
        torch.cuda.synchronize()
        clk.mark_end()
        barrier(world)
    gms = max_over_ranks(gs.elapsed_time(ge), world)
    del g
    return {"ms_per_step": gms / steps, "elapsed_ms": gms}, clk.summary()


def run_workload(wl, name, args, steps, world, local, hbm, tf_burst, tf_sust, peak_kind):
    """Time one workload: K eager steps with CUDA events around every gate_up
    launch (the dominant kernel), then the same steps as one CUDA graph.
    Returns the workload's entry (value = graphed layer-tokens/s)."""
    shape, T, layers = wl.shape, wl.T, wl.L
    stream = torch.cuda.current_stream()
    for _ in range(max(args.warmup, 3)):
        wl.step(args.algo)
    torch.cuda.synchronize()

    n_ev = 4 if (args.lora or args.backward) else 2
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
            for _ in range(layers)] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        clk.mark_start()
        start.record(stream)
        for s in range(steps):
            wl.step(args.algo, evs[s])
        end.record(stream)
        torch.cuda.synchronize()
        clk.mark_end()
        barrier(world)
    elapsed_ms = max_over_ranks(start.elapsed_time(end), world)
    tokens_per_step = T * layers          # layer-tokens: T tokens through each layer
    eager_value = world * tokens_per_step * steps / (elapsed_ms / 1e3)
    gu_ms = [e[0].elapsed_time(e[1]) for st in evs for e in st]
    gu_avg_ms = sum(gu_ms) / len(gu_ms)
    lora_ms = [e[2].elapsed_time(e[3]) for st in evs for e in st] if args.lora else []

    d = wl.distinct_experts()
    d_avg = sum(d) / len(d)
    gu_bytes = sum(wl.gate_up_bytes(x) for x in d) / len(d)
    gu_flops = wl.gate_up_flops()
    # the tensor-core kernel serves the GEMMs from 36 routed rows per expert
    # on average (the AUTO dispatch rule); below that the decode GEMV does
    prefill = T * shape.k >= 36 * shape.E and args.algo != "gemv"
    epi_name = "(fp32 out)" if (args.lora or args.backward) else "+ SwiGLU"
    workload_key = f"{name}:T={T}"
    if prefill:
        achieved = gu_flops / (gu_avg_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tf_burst, "unit": "TFLOP/s",
                "frac": achieved / tf_burst,
                "frac_of_nominal": achieved / NOMINAL_BF16_TFLOPS,
                "traffic": recorded_traffic("grouped_gemm_tc.cu", workload_key),
                "kernel": f"grouped {args.weights.upper()} gate_up GEMM {epi_name} (tcgen05)",
                "per_launch": f"{gu_flops:.4g} FLOP (2*T*k*H*2I, real routed rows)",
                "us_per_launch": 1e3 * gu_avg_ms,
                "peak_source": f"{peak_kind} bf16 dense (burst); nominal "
                               f"{NOMINAL_BF16_TFLOPS:.0f} for frac_of_nominal"}
    else:
        achieved = gu_bytes / (gu_avg_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
                "traffic": recorded_traffic(DECODE_KERNEL_SOURCE[args.weights], workload_key),
                "kernel": f"grouped {args.weights.upper()} gate_up GEMV {epi_name}",
                "per_launch": f"{gu_bytes:.4g} B (distinct experts {d_avg:.1f} x 2I*H*"
                              f"{BYTES_PER_WEIGHT[args.weights]} + X + output)",
                "us_per_launch": 1e3 * gu_avg_ms,
                "peak_source": f"{peak_kind} HBM copy; nominal {NOMINAL_HBM_GBS:.0f} for "
                               "frac_of_nominal"}

    graphed, gclk = graphed_replay(wl, args.algo, steps, args.warmup, world, local)
    entry = {"workload": name, "T": T, "layers": layers}
    if "ms_per_step" in graphed:
        entry["value"] = world * tokens_per_step * steps / (graphed["elapsed_ms"] / 1e3)
        entry["ms_per_step"] = graphed["ms_per_step"]
        entry["clocks"] = gclk
        entry["timing"] = "graphed"
    else:
        entry["value"] = eager_value
        entry["ms_per_step"] = elapsed_ms / steps
        entry["clocks"] = clk.summary()
        entry["timing"] = f"eager (graph capture failed: {graphed.get('error')})"
    entry["unit"] = "layer-tokens/s"
    entry["eager"] = {"value": eager_value, "ms_per_step": elapsed_ms / steps,
                      "clocks": clk.summary()}
    entry["roofline"] = roof
    entry["distinct_experts_per_layer"] = d_avg
    layer_ms = entry["ms_per_step"] / layers
    if not prefill:
        # the whole layer against the decode bytes it must move
        lb = sum(wl.layer_bytes(x) for x in d) / len(d)
        entry["layer_hbm"] = {"bytes_per_layer": lb, "us_per_layer": 1e3 * layer_ms,
                              "achieved_GBs": lb / (layer_ms / 1e3) / 1e9,
                              "frac": lb / (layer_ms / 1e3) / 1e9 / hbm}
    else:
        lf = 3 * gu_flops / 2
        entry["layer_tensor"] = {"flops_per_layer": lf, "us_per_layer": 1e3 * layer_ms,
                                 "achieved_TFLOPs": lf / (layer_ms / 1e3) / 1e12,
                                 "frac": lf / (layer_ms / 1e3) / 1e12 / tf_burst}
    entry["tokens_per_s_through_all_layers"] = world * T / (layer_ms * layers / 1e3)
    entry["gate_up_ms_avg"] = gu_avg_ms
    if args.lora:
        lb = sum(wl.lora_bytes(x) for x in d) / len(d)
        l_avg = sum(lora_ms) / len(lora_ms)
        lach = lb / (l_avg / 1e3) / 1e9
        entry["lora"] = {"rank": args.lora, "kernel": "gate_up LoRA delta (in place on fp32)",
                         "timing": "CUDA events around each eager launch; at decode sizes the "
                                   "window can include the wait for the host to submit it",
                         "us_per_launch": 1e3 * l_avg, "bytes_per_launch": lb,
                         "per_launch": f"distinct experts {d_avg:.1f} x r*(H+2I)*2 + X + 2 x "
                                       "fp32 out",
                         "achieved_GBs": lach, "frac_of_hbm": lach / hbm,
                         "flops_per_launch": 2.0 * T * shape.k * args.lora
                                             * (shape.H + 2 * shape.I)}
    return entry


def cpu_baseline_for(shape, T, name, args, cache):
    """The oracle on the host cores on a bounded sample of this workload's
    tokens (rank 0 at N = 1 only); one sample per shape serves every batch
    size of that shape, since the oracle's cost per token does not depend on
    the batch."""
    key = (shape.name, args.weights)
    if key in cache:
        out = dict(cache[key])
        out["sample"] = out["sample"] + f" (measured on {out['measured_on']}, reused)"
        return out
    ncpu, aff, threads = cpu_cores()
    n_tok = min(T, 16 if shape.H <= 256 else 4 if shape.H <= 2048 else 2)
    n, dt = oracle_sample(shape, T, args.seed, n_tok, weights=args.weights)
    cpu = {"value": n / dt, "unit": "layer-tokens/s", "cores": threads, "kind": "oracle",
           "blas_threads": threads, "measured_on": f"{name}:T={T}",
           "sample": f"{n} tokens of layer 0 (their experts dequantized, per-token fp64 "
                     f"expert MLPs); host cpu_count={ncpu}, affinity={aff}; {dt:.2f} s"}
    try:  # the same oracle on one thread
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            n1, dt1 = oracle_sample(shape, T, args.seed, max(1, n_tok // 2), weights=args.weights)
        cpu["value_1thread"] = n1 / dt1
        cpu["sample"] += f"; 1-thread run: {n1} tokens in {dt1:.2f} s"
    except ImportError:
        pass
    cache[key] = cpu
    return dict(cpu)


# ----------------------------------------------------------------- main

def main():
    args = parse_args()
    shape, T, layers = CONFIGS[args.config]
    T = args.tokens or T
    layers = args.layers or layers
    if args.impl == "reference":
        run_reference(args, shape, T, layers)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device for --impl ours")
    world, rank, local = dist_setup()
    import bit_mixture_experts_route_b200 as moe
    moe.load()
    if args.backward and args.weights != "nf4":
        raise SystemExit("--backward runs on NF4 weights (the transposed GEMM is NF4)")
    hbm, tf_burst, tf_sust, peak_kind = load_peaks()
    seed = rank_seed(args.seed, rank)
    wl = Workload(shape, T, layers, seed, weights=args.weights, lora=args.lora,
                  backward=args.backward)
    wl_tc_backward = args.backward and wl.tc_backward()
    workload_name = (args.config + (f"/{args.weights}" if args.weights != "nf4" else "")
                     + (f"/lora-r{args.lora}" if args.lora else "")
                     + ("/fwd+bwd" if args.backward else ""))
    head = run_workload(wl, workload_name, args, args.steps, world, local, hbm, tf_burst,
                        tf_sust, peak_kind)

    # ---- end to end through the one-call C API with host buffers: every
    # step copies its inputs from pinned host memory and its output back.
    # The plain NF4 layer runs two steps in flight (double-buffered inputs and
    # output; uploads and downloads on two more streams, so PCIe runs both
    # directions at once), as a serving loop overlaps the next batch's upload
    # and the last batch's download with the current compute; the other paths
    # copy and compute on one stream.
    X_h = wl.X.cpu().pin_memory()
    L_h = wl.logits.cpu().pin_memory()
    pipelined = wl.fmt == "nf4" and not (wl.lora or wl.backward)
    nbuf = 2 if pipelined else 1
    Y_h = [torch.empty((T, shape.H), dtype=torch.float32).pin_memory() for _ in range(nbuf)]
    X_d = [torch.empty_like(wl.X) for _ in range(nbuf)]
    L_d = [torch.empty_like(wl.logits) for _ in range(nbuf)]
    Y_d = [torch.empty((T, shape.H), dtype=torch.float32, device=wl.X.device)
           for _ in range(nbuf)]
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(nbuf)]
    ev_out = [torch.cuda.Event() for _ in range(nbuf)]
    ev_free = [torch.cuda.Event() for _ in range(nbuf)]

    def e2e_step(s):
        b = s % nbuf
        if not pipelined:  # the calls one by one, copies on the compute stream
            X_d[0].copy_(X_h, non_blocking=True)
            L_d[0].copy_(L_h, non_blocking=True)
            for layer in range(layers):
                wl.layer(layer, args.algo, X=X_d[0], logits=L_d[0][layer])
            Y_h[0].copy_(wl.Y, non_blocking=True)
            return
        with torch.cuda.stream(up):
            up.wait_event(ev_free[b])  # step s - 2 is done with buffer b
            X_d[b].copy_(X_h, non_blocking=True)
            L_d[b].copy_(L_h, non_blocking=True)
            ev_in[b].record(up)
        comp.wait_event(ev_in[b])
        for layer in range(layers):
            moe.layer_forward(X_d[b], L_d[b][layer], shape.k, shape.renormalize,
                              *wl.stacks[layer], workspace=wl.lws, out=Y_d[b])
        ev_out[b].record(comp)
        with torch.cuda.stream(down):
            down.wait_event(ev_out[b])
            Y_h[b].copy_(Y_d[b], non_blocking=True)
            ev_free[b].record(down)

    for s in range(3):
        e2e_step(s)
    torch.cuda.synchronize()
    es, ee = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    es.record(comp)
    for s in range(args.steps):
        e2e_step(3 + s)
    comp.wait_stream(down)  # the last step's output is on the host
    ee.record(comp)
    torch.cuda.synchronize()
    ems = max_over_ranks(es.elapsed_time(ee), world)
    e2e = {"value": world * T * layers * args.steps / (ems / 1e3), "unit": "tokens/s",
           "h2d_bytes_per_step": X_h.numel() * 2 + L_h.numel() * 4,
           "d2h_bytes_per_step": Y_h[0].numel() * 4,
           "path": ("moe_layer_forward per layer (C ABI), pinned host X and logits in, Y out; "
                    + ("two steps in flight, uploads and downloads on their own streams"
                       if pipelined
                       else "copies and compute on one stream"))}
    del wl
    torch.cuda.empty_cache()

    baselines = {}
    cpu = None
    do_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    if (args.lora or args.backward) and not args.no_cpu_baseline:
        cpu = {"skipped": "the oracle's timed layer is the plain forward; the adapter and "
                          "backward oracles are checked in the tests"}
    elif do_cpu:
        cpu = cpu_baseline_for(shape, T, workload_name, args, baselines)

    # ---- the rest of the workload list (same collective steps on every rank)
    workloads = []
    plain = args.weights == "nf4" and not args.lora and not args.backward
    if plain and not args.no_sweep and args.config == HEADLINE and args.tokens is None \
            and args.layers is None:
        sweep_steps = min(args.steps, SWEEP_STEPS)
        current = None
        for cfg, t in SWEEP:
            sh, _, nl = CONFIGS[cfg]
            if current is None or current[0] != cfg:
                current = None
                torch.cuda.empty_cache()
                current = (cfg, Workload(sh, t, nl, seed))
            w = current[1]
            print(f"[bench] {cfg} T={t}", file=sys.stderr, flush=True)
            w.set_tokens(t)
            entry = run_workload(w, cfg, args, sweep_steps, world, local, hbm, tf_burst,
                                 tf_sust, peak_kind)
            if do_cpu:
                entry["cpu_baseline"] = cpu_baseline_for(sh, t, cfg, args, baselines)
            entry["config"] = {"E": sh.E, "k": sh.k, "hidden": sh.H, "intermediate": sh.I,
                               "renormalize": sh.renormalize, "routing": sh.routing,
                               "l2": f"{nl} layers x {sh.E * sh.nf4_bytes_per_expert / 1e6:.1f}"
                                     " MB NF4 weights"}
            workloads.append(entry)
        current = None
        torch.cuda.empty_cache()

    # route_tile, permute_scatter, permute_rows, gate_up, down, combine; the
    # standalone SwiGLU when adapted or with the backward; two adapter
    # launches; the backward's combine backward, two transposed GEMMs, SwiGLU
    # backward, scatter-add and routing backward
    launches_per_layer = (6 + (1 if (args.lora or args.backward) else 0) + (2 if args.lora else 0)
                          + (6 if args.backward else 0))
    if args.backward and wl_tc_backward:
        launches_per_layer -= 1     # the fused down + SwiGLU backward
    line = {
        "metric": "MoE layer tokens/s", "value": head["value"], "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": workload_name, "T": T, "layers": layers, "E": shape.E,
                   "k": shape.k, "hidden": shape.H, "intermediate": shape.I,
                   "weights": args.weights, "renormalize": shape.renormalize,
                   "routing": shape.routing,
                   "value_counts": "layer-tokens: T tokens through each of the layers",
                   "l2": f"inputs larger than L2: {layers} layers x "
                         f"{shape.E * shape.nf4_bytes_per_expert / 1e6:.0f} MB NF4 weights",
                   "distinct_experts_per_layer": head["distinct_experts_per_layer"],
                   "algo": args.algo,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "roofline": head["roofline"],
        "timing": "value = the layer steps replayed as one CUDA graph of moe_layer_forward "
                  "calls (the library's chained launches); eager = the exported calls one by "
                  "one from the host, CUDA events around each gate_up launch",
        "graphed": {"value": head["value"], "ms_per_step": head["ms_per_step"]}
        if head["timing"] == "graphed" else {"error": head["timing"]},
        "eager": head["eager"],
        "e2e": e2e,
        "cpu_baseline": cpu,
        "gpu_launches": launches_per_layer * layers * args.steps,
        "clocks": head["clocks"],
        "gate_up_ms_avg": head["gate_up_ms_avg"],
    }
    for key in ("layer_hbm", "layer_tensor", "lora"):
        if key in head:
            line[key] = head[key]
    if workloads:
        line["workloads"] = workloads
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
