"""Routing without a caller-provided workspace (moe_route_permute_noalloc).

Callers that cannot allocate device memory where they route -- a host
framework that owns all device memory through its own allocator, or a
latency-critical loop where cudaMalloc may synchronize the device -- use this
entry point; its scratch is a fixed array inside the library.  These tests
check, through the C ABI, that it returns exactly what moe_route_permute
returns with a workspace, on two calls in a row (the second reuses the
scratch the first left behind), and that oversized problems are refused.

This file is collected last on purpose.
"""

import ctypes

import numpy as np
import pytest
import torch

from bit_mixture_experts_route_b200 import _lib

MAX_BYTES = 1 << 20  # MOE_ROUTE_NOALLOC_SCRATCH_BYTES


def _noalloc(logits, k, renorm):
    T, E = logits.shape
    dev = logits.device
    out = {
        "topk_idx": torch.empty((T, k), dtype=torch.int32, device=dev),
        "topk_w": torch.empty((T, k), dtype=torch.float32, device=dev),
        "expert_offsets": torch.empty((E + 1,), dtype=torch.int32, device=dev),
        "sorted_rows": torch.empty((T * k,), dtype=torch.int32, device=dev),
        "inv_perm": torch.empty((T * k,), dtype=torch.int32, device=dev),
    }
    st = _lib.load().moe_route_permute_noalloc(
        _lib._ptr(logits), T, E, k, 1 if renorm else 0, _lib._ptr(out["topk_idx"]),
        _lib._ptr(out["topk_w"]), _lib._ptr(out["expert_offsets"]),
        _lib._ptr(out["sorted_rows"]), _lib._ptr(out["inv_perm"]), _lib._stream(dev))
    assert st == 0, _lib.STATUS.get(st, st)
    return out


@pytest.mark.gpu
def test_noalloc_routing_matches_workspace_routing_twice():
    import bit_mixture_experts_route_b200 as moe
    g = torch.Generator().manual_seed(123)
    # A large call first (32768 routed rows), then a smaller one (4800 rows)
    # that also takes the two-launch path through the scratch, so it runs on
    # the ranks and tile counts the large call left behind.  Both sizes lie
    # above the 4096 routed rows that the one-launch path (which needs no
    # scratch) handles.
    cases = [(4096, 128, 8, True), (600, 64, 8, False)]
    for T, E, k, renorm in cases:
        logits = torch.randn((T, E), generator=g).cuda()
        ref = moe.route_permute(logits, k, renorm)
        got = _noalloc(logits, k, renorm)
        torch.cuda.synchronize()
        for key in ("topk_idx", "expert_offsets", "sorted_rows", "inv_perm"):
            assert torch.equal(got[key], ref[key]), key
        np.testing.assert_allclose(got["topk_w"].cpu().numpy(), ref["topk_w"].cpu().numpy(),
                                   rtol=2e-6, atol=1e-9)
        assert got["sorted_rows"].numel() == T * k


def test_noalloc_routing_refuses_oversized_problems():
    # Rejected on the host before any CUDA call (fake, never-used addresses).
    lib = _lib.load()
    a = ctypes.c_void_p(0x7000_0000)
    T, E, k = 40000, 128, 8
    assert _lib.route_permute_workspace_size(T, E, k) > MAX_BYTES
    st = lib.moe_route_permute_noalloc(a, T, E, k, 1, a, a, a, a, a, None)
    assert st == 4  # MOE_ERR_WORKSPACE
