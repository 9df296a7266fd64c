"""The Python binding rejects buffers the kernels would overrun, before any
library call (CPU: tensors are presented as device tensors and the library is
a recorder that must stay unused)."""

import pytest
import torch

from bit_mixture_experts_route_b200 import _lib


class _Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def f(*args):
            self.calls.append(name)
            return 0
        return f


@pytest.fixture
def lib(monkeypatch):
    rec = _Recorder()
    monkeypatch.setattr(torch.Tensor, "is_cuda", property(lambda self: True))
    monkeypatch.setattr(_lib, "_lib", rec)
    monkeypatch.setattr(_lib, "_stream", lambda device=None: None)
    return rec


def test_room_checks_size_contiguity_and_dtype(lib):
    _lib._room(torch.empty(10), 10, "x")
    with pytest.raises(_lib.MoEError, match="needs 11"):
        _lib._room(torch.empty(10), 11, "x")
    with pytest.raises(_lib.MoEError, match="contiguous"):
        _lib._room(torch.empty(4, 4).t(), 4, "x")
    with pytest.raises(_lib.MoEError, match="one of"):
        _lib._room(torch.empty(4, dtype=torch.int32), 4, "x", (torch.float32,))


def _nf4(E=2, N=128, K=256):
    return (torch.zeros((E, N, K // 2), dtype=torch.uint8),
            torch.zeros((E, N * K // 64), dtype=torch.float32))


def test_grouped_gemm_rejects_small_out_offsets_and_absmax(lib):
    packed, absmax = _nf4()
    A = torch.zeros((8, 256), dtype=torch.float16)
    off = torch.zeros(3, dtype=torch.int32)
    _lib.nf4_grouped_gemm(A, packed, absmax, off, 8)            # well-formed: reaches the library
    assert lib.calls == ["moe_nf4_grouped_gemm"]
    with pytest.raises(_lib.MoEError, match="out"):
        _lib.nf4_grouped_gemm(A, packed, absmax, off, 8, out=torch.empty((7, 128)))
    with pytest.raises(_lib.MoEError, match="expert_offsets"):
        _lib.nf4_grouped_gemm(A, packed, absmax, off[:2], 8)
    with pytest.raises(_lib.MoEError, match="absmax"):
        _lib.nf4_grouped_gemm(A, packed, absmax[:, :-1].contiguous(), off, 8)
    with pytest.raises(_lib.MoEError, match="gather"):
        _lib.nf4_grouped_gemm(A, packed, absmax, off, 8,
                              gather=torch.zeros(7, dtype=torch.int32), k=2)
    assert lib.calls == ["moe_nf4_grouped_gemm"]


def test_combine_and_routing_calls_reject_mismatched_rows(lib):
    T, k, H, E = 4, 2, 16, 8
    w = torch.zeros((T, k))
    inv = torch.zeros(T * k, dtype=torch.int32)
    with pytest.raises(_lib.MoEError, match="Yp"):
        _lib.unpermute_combine(torch.zeros((T * k - 1, H)), inv, w)
    with pytest.raises(_lib.MoEError, match="inv_perm"):
        _lib.unpermute_combine(torch.zeros((T * k, H)), inv[:-1], w)
    with pytest.raises(_lib.MoEError, match="dY"):
        _lib.combine_backward(torch.zeros((T + 1, H)), torch.zeros((T * k, H)), inv, w)
    with pytest.raises(_lib.MoEError, match="dw"):
        _lib.route_backward(torch.zeros((T, E)), torch.zeros((T, k), dtype=torch.int32), w,
                            torch.zeros((T, k + 1)), True)
    out = {"topk_idx": torch.zeros((T, k), dtype=torch.int32), "topk_w": w,
           "expert_offsets": torch.zeros(E, dtype=torch.int32),       # one short
           "sorted_rows": inv, "inv_perm": inv}
    with pytest.raises(_lib.MoEError, match="expert_offsets"):
        _lib.route_permute(torch.zeros((T, E)), k, True, workspace=torch.zeros(256, dtype=torch.uint8),
                           out=out)
    assert lib.calls == []


def test_layer_forward_rejects_short_stacks(lib):
    T, E, k, H, I = 4, 8, 2, 256, 128
    X = torch.zeros((T, H), dtype=torch.bfloat16)
    lg = torch.zeros((T, E))
    p_gu = torch.zeros((E, 2 * I, H // 2), dtype=torch.uint8)
    a_gu = torch.zeros((E, 2 * I * H // 64))
    p_d = torch.zeros((E, H, I // 2), dtype=torch.uint8)
    a_d = torch.zeros((E, H * I // 64))
    with pytest.raises(_lib.MoEError, match="absmax_d"):
        _lib.layer_forward(X, lg, k, True, p_gu, a_gu, p_d, a_d[:-1])
    with pytest.raises(_lib.MoEError, match="logits"):
        _lib.layer_forward(X, lg[:-1], k, True, p_gu, a_gu, p_d, a_d)
    assert "moe_layer_forward" not in lib.calls
