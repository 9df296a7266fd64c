"""ctypes binding of libmoenf4.so: argument marshalling only.

Every function here takes torch CUDA tensors, checks dtype / shape /
contiguity, allocates outputs with torch when the caller does not pass them,
and calls the C entry point of the same name on the current CUDA stream.
All arithmetic runs in the library's kernels; there is no fallback.  If the
shared library is missing, importing any op raises.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoenf4.so")

MOE_OK = 0
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_MISALIGNED",
          3: "MOE_ERR_UNSUPPORTED", 4: "MOE_ERR_WORKSPACE", 5: "MOE_ERR_CUDA"}
DT = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}
EPI = {"none": 0, "swiglu": 1}
ALGO = {"auto": 0, "gemv": 1, "tc": 2, "tc_pair": 3}
DEVERR_NONFINITE, DEVERR_BAD_OFFSETS, DEVERR_BAD_INDEX, DEVERR_TIMEOUT = 1, 2, 4, 8
DEVERR_LAYOUT, DEVERR_RANGE = 0x10, 0x20

# Every exported symbol with (restype, argtypes); the header declares them.
_P, _I, _Z, _S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
SIGNATURES = {
    "moe_status_string": (ctypes.c_char_p, [_I]),
    "moe_abi_version": (_I, []),
    "moe_last_cuda_error": (ctypes.c_char_p, []),
    "moe_nf4_levels": (_I, [_P]),
    "moe_nf4_quantize": (_I, [_P, _I, _I, _I, _I, _P, _P, _P, _S]),
    "moe_nf4_dequantize": (_I, [_P, _P, _I, _I, _I, _P, _I, _S]),
    "moe_route_permute_workspace_size": (_I, [_I, _I, _I, ctypes.POINTER(ctypes.c_size_t)]),
    "moe_route_permute": (_I, [_P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _Z, _S]),
    "moe_route_permute_noalloc": (_I, [_P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _S]),
    "moe_nf4_grouped_gemm": (_I, [_P, _I, _I, _P, _I, _P, _P, _P, _I, _I, _I, _I, _I, _P,
                                  _I, _I, _P, _S]),
    "moe_int4_quantize": (_I, [_P, _I, _I, _I, _P, _P, _P, _S]),
    "moe_int4_grouped_gemm": (_I, [_P, _I, _P, _P, _P, _I, _I, _I, _I, _I, _P, _I, _I, _P, _S]),
    "moe_mxfp4_quantize": (_I, [_P, _I, _I, _I, _P, _P, _P, _S]),
    "moe_mxfp4_grouped_gemm": (_I, [_P, _I, _P, _P, _P, _I, _I, _I, _I, _I, _P, _I, _I, _P,
                                    _S]),
    "moe_nf4_grouped_gemm_t": (_I, [_P, _I, _I, _P, _P, _P, _I, _I, _I, _I, _P, _I, _I, _P,
                                    _S]),
    "moe_nf4_down_backward": (_I, [_P, _I, _P, _P, _P, _I, _I, _I, _I, _P, _P, _I, _P, _S]),
    "moe_swiglu_backward": (_I, [_P, _P, _I, _I, _I, _P, _I, _S]),
    "moe_combine_backward": (_I, [_P, _P, _I, _P, _P, _I, _I, _I, _P, _I, _P, _P, _S]),
    "moe_route_backward": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _S]),
    "moe_lora_delta": (_I, [_P, _I, _P, _I, _I, _I, _I, _P, _P, ctypes.c_float, _I, _P, _P, _S]),
    "moe_permute_rows": (_I, [_P, _I, _I, _I, _P, _I, _I, _P, _P, _S]),
    "moe_swiglu": (_I, [_P, _I, _I, _I, _P, _I, _S]),
    "moe_unpermute_combine": (_I, [_P, _I, _P, _P, _I, _I, _I, _P, _I, _S]),
    "moe_layer_workspace_size": (_I, [_I, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_size_t)]),
    "moe_layer_forward": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _Z,
                               _P, _S]),
}

_lib = None


class MoEError(RuntimeError):
    pass


def load() -> ctypes.CDLL:
    """Load libmoenf4.so (once) and bind every exported signature."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise MoEError(f"{LIB_PATH} is missing: build it with "
                           "`python -m bit_mixture_experts_route_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _check(status: int, what: str):
    if status != MOE_OK:
        detail = ""
        if status == 5:
            detail = f" ({load().moe_last_cuda_error().decode()})"
        raise MoEError(f"{what}: {STATUS.get(status, status)}{detail}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t, dtype, name, ndim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise MoEError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise MoEError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise MoEError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise MoEError(f"{name} must have {ndim} dims")


def _room(t, n, name, dtypes=None):
    """``t`` is a contiguous CUDA tensor (of one of ``dtypes``) with at least
    ``n`` elements: the kernels address that many, so a smaller buffer would
    be read or written out of bounds on the device."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise MoEError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise MoEError(f"{name} must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise MoEError(f"{name} must be one of {dtypes}, got {t.dtype}")
    if t.numel() < n:
        raise MoEError(f"{name} has {t.numel()} elements, the call needs {n}")


_F = (torch.float32, torch.bfloat16, torch.float16)


def nf4_levels():
    buf = (ctypes.c_float * 16)()
    _check(load().moe_nf4_levels(ctypes.cast(buf, ctypes.c_void_p)), "moe_nf4_levels")
    return list(buf)


def nf4_quantize(W, packed=None, absmax=None, dev_err=None):
    """``W fp32 [E, N, K]`` -> ``(packed u8 [E, N, K/2], absmax fp32 [E, N*K/64])``."""
    _need(W, torch.float32, "W", 3)
    E, N, K = W.shape
    if packed is None:
        packed = torch.empty((E, N, K // 2), dtype=torch.uint8, device=W.device)
    if absmax is None:
        absmax = torch.empty((E, N * K // 64), dtype=torch.float32, device=W.device)
    _room(packed, E * N * (K // 2), "packed", (torch.uint8,))
    _room(absmax, E * N * (K // 64), "absmax", (torch.float32,))
    _check(load().moe_nf4_quantize(_ptr(W), E, N, K, 64, _ptr(packed), _ptr(absmax),
                                   _ptr(dev_err), _stream(W.device)), "moe_nf4_quantize")
    return packed, absmax


def nf4_dequantize(packed, absmax, out_dtype=torch.float32):
    _need(packed, torch.uint8, "packed", 3)
    E, N, half = packed.shape
    _room(absmax, E * N * (2 * half // 64), "absmax", (torch.float32,))
    out = torch.empty((E, N, 2 * half), dtype=out_dtype, device=packed.device)
    _check(load().moe_nf4_dequantize(_ptr(packed), _ptr(absmax), E, N, 2 * half, _ptr(out),
                                     DT[out_dtype], _stream(packed.device)),
           "moe_nf4_dequantize")
    return out


def route_permute_workspace_size(T, E, k):
    n = ctypes.c_size_t()
    _check(load().moe_route_permute_workspace_size(T, E, k, ctypes.byref(n)),
           "moe_route_permute_workspace_size")
    return n.value


def route_permute(logits, k, renormalize=True, workspace=None, out=None):
    """``logits fp32 [T, E]`` -> dict of topk_idx, topk_w, expert_offsets,
    sorted_rows, inv_perm (device tensors)."""
    _need(logits, torch.float32, "logits", 2)
    T, E = logits.shape
    dev = logits.device
    if out is None:
        out = {
            "topk_idx": torch.empty((T, k), dtype=torch.int32, device=dev),
            "topk_w": torch.empty((T, k), dtype=torch.float32, device=dev),
            "expert_offsets": torch.empty((E + 1,), dtype=torch.int32, device=dev),
            "sorted_rows": torch.empty((T * k,), dtype=torch.int32, device=dev),
            "inv_perm": torch.empty((T * k,), dtype=torch.int32, device=dev),
        }
    for key, n, dt in (("topk_idx", T * k, torch.int32), ("topk_w", T * k, torch.float32),
                       ("expert_offsets", E + 1, torch.int32), ("sorted_rows", T * k, torch.int32),
                       ("inv_perm", T * k, torch.int32)):
        _room(out[key], n, key, (dt,))
    nbytes = route_permute_workspace_size(T, E, k)
    if workspace is None:
        workspace = torch.empty((max(nbytes, 256),), dtype=torch.uint8, device=dev)
    _room(workspace, 0, "workspace")
    _check(load().moe_route_permute(
        _ptr(logits), T, E, k, 1 if renormalize else 0, _ptr(out["topk_idx"]),
        _ptr(out["topk_w"]), _ptr(out["expert_offsets"]), _ptr(out["sorted_rows"]),
        _ptr(out["inv_perm"]), _ptr(workspace), workspace.numel(), _stream(dev)),
        "moe_route_permute")
    return out


def nf4_grouped_gemm(A, packed, absmax, expert_offsets, M_total, gather=None, k=1,
                     epilogue="none", out_dtype=torch.float32, algo="auto", out=None,
                     dev_err=None):
    """Grouped NF4 GEMM over all experts in one launch (see the header)."""
    if A.dtype not in (torch.bfloat16, torch.float16):
        raise MoEError("A must be bf16 or fp16")
    _need(A, A.dtype, "A", 2)
    _need(packed, torch.uint8, "packed", 3)
    _need(absmax, torch.float32, "absmax")
    _need(expert_offsets, torch.int32, "expert_offsets", 1)
    E, N, half = packed.shape
    K = 2 * half
    if A.shape[1] != K:
        raise MoEError("A's columns must equal the weights' K")
    if gather is not None:
        _need(gather, torch.int32, "gather", 1)
        _room(gather, M_total, "gather")
    _room(absmax, E * N * (K // 64), "absmax")
    _room(expert_offsets, E + 1, "expert_offsets")
    n_out = N // 2 if epilogue == "swiglu" else N
    if out is None:
        out = torch.empty((M_total, n_out), dtype=out_dtype, device=A.device)
    _room(out, M_total * n_out, "out", _F)
    _check(load().moe_nf4_grouped_gemm(
        _ptr(A), DT[A.dtype], A.shape[0], _ptr(gather), k, _ptr(packed), _ptr(absmax),
        _ptr(expert_offsets), E, N, K, M_total, EPI[epilogue], _ptr(out), DT[out.dtype],
        ALGO[algo], _ptr(dev_err), _stream(A.device)), "moe_nf4_grouped_gemm")
    return out


def int4_quantize(W, packed=None, meta=None, dev_err=None):
    """``W fp32 [E, N, K]`` -> ``(packed u8 [E, N, K/2], meta u32-as-int32
    [E, N, K/128])``: grouped INT4 codes, per 128-group fp16 scale | zero << 16."""
    _need(W, torch.float32, "W", 3)
    E, N, K = W.shape
    if packed is None:
        packed = torch.empty((E, N, K // 2), dtype=torch.uint8, device=W.device)
    if meta is None:
        meta = torch.empty((E, N, K // 128), dtype=torch.int32, device=W.device)
    _room(packed, E * N * (K // 2), "packed", (torch.uint8,))
    _room(meta, E * N * (K // 128), "meta", (torch.int32,))
    _check(load().moe_int4_quantize(_ptr(W), E, N, K, _ptr(packed), _ptr(meta), _ptr(dev_err),
                                    _stream(W.device)), "moe_int4_quantize")
    return packed, meta


def int4_grouped_gemm(A, packed, meta, expert_offsets, M_total, epilogue="none",
                      out_dtype=torch.float32, out=None, dev_err=None, algo="auto"):
    """Grouped GEMM on INT4 weights, all experts in one launch (decode GEMV or
    tensor-core kernel, see the header); ``A`` fp16 rows in permuted order."""
    _need(A, torch.float16, "A", 2)
    _need(packed, torch.uint8, "packed", 3)
    _need(meta, torch.int32, "meta", 3)
    _need(expert_offsets, torch.int32, "expert_offsets", 1)
    E, N, half = packed.shape
    K = 2 * half
    if A.shape[1] != K:
        raise MoEError("A's columns must equal the weights' K")
    _room(meta, E * N * (K // 128), "meta")
    _room(expert_offsets, E + 1, "expert_offsets")
    n_out = N // 2 if epilogue == "swiglu" else N
    if out is None:
        out = torch.empty((M_total, n_out), dtype=out_dtype, device=A.device)
    _room(out, M_total * n_out, "out", _F)
    _check(load().moe_int4_grouped_gemm(
        _ptr(A), A.shape[0], _ptr(packed), _ptr(meta), _ptr(expert_offsets), E, N, K, M_total,
        EPI[epilogue], _ptr(out), DT[out.dtype], ALGO[algo], _ptr(dev_err), _stream(A.device)),
        "moe_int4_grouped_gemm")
    return out


def mxfp4_quantize(W, packed=None, scales=None, dev_err=None):
    """``W fp32 [E, N, K]`` -> ``(packed u8 [E, N, K/2], scales u8 [E, N, K/32])``:
    E2M1 codes (element 2j in the low nibble) and E8M0 scale bytes."""
    _need(W, torch.float32, "W", 3)
    E, N, K = W.shape
    if packed is None:
        packed = torch.empty((E, N, K // 2), dtype=torch.uint8, device=W.device)
    if scales is None:
        scales = torch.empty((E, N, K // 32), dtype=torch.uint8, device=W.device)
    _room(packed, E * N * (K // 2), "packed", (torch.uint8,))
    _room(scales, E * N * (K // 32), "scales", (torch.uint8,))
    _check(load().moe_mxfp4_quantize(_ptr(W), E, N, K, _ptr(packed), _ptr(scales), _ptr(dev_err),
                                     _stream(W.device)), "moe_mxfp4_quantize")
    return packed, scales


def mxfp4_grouped_gemm(A, packed, scales, expert_offsets, M_total, epilogue="none",
                       out_dtype=torch.float32, algo="auto", out=None, dev_err=None):
    """Grouped GEMM on MXFP4 weights, all experts in one launch (decode GEMV
    or tensor-core kernel, see the header); ``A`` fp16 rows in permuted
    order."""
    _need(A, torch.float16, "A", 2)
    _need(packed, torch.uint8, "packed", 3)
    _need(scales, torch.uint8, "scales", 3)
    _need(expert_offsets, torch.int32, "expert_offsets", 1)
    E, N, half = packed.shape
    K = 2 * half
    if A.shape[1] != K or scales.shape != (E, N, K // 32):
        raise MoEError("A's columns and the scales must match the weights' K")
    _room(expert_offsets, E + 1, "expert_offsets")
    n_out = N // 2 if epilogue == "swiglu" else N
    if out is None:
        out = torch.empty((M_total, n_out), dtype=out_dtype, device=A.device)
    _room(out, M_total * n_out, "out", _F)
    _check(load().moe_mxfp4_grouped_gemm(
        _ptr(A), A.shape[0], _ptr(packed), _ptr(scales), _ptr(expert_offsets), E, N, K, M_total,
        EPI[epilogue], _ptr(out), DT[out.dtype], ALGO[algo], _ptr(dev_err), _stream(A.device)),
        "moe_mxfp4_grouped_gemm")
    return out


def nf4_grouped_gemm_t(G, packed, absmax, expert_offsets, M_total, out_dtype=torch.float32,
                       out=None, dev_err=None, algo="auto"):
    """Transposed grouped NF4 GEMM: ``out[p] = W[e(p)]^T @ G[p]`` -> ``[M_total, K]``;
    ``G`` fp32 or fp16 ``[>= M_total, N]`` (the backward of ``nf4_grouped_gemm``)."""
    if G.dtype not in (torch.float32, torch.float16):
        raise MoEError("G must be fp32 or fp16")
    _need(G, G.dtype, "G", 2)
    _need(packed, torch.uint8, "packed", 3)
    _need(absmax, torch.float32, "absmax")
    _need(expert_offsets, torch.int32, "expert_offsets", 1)
    E, N, half = packed.shape
    K = 2 * half
    if G.shape[1] != N:
        raise MoEError("G's columns must equal the weights' N")
    _room(absmax, E * N * (K // 64), "absmax")
    _room(expert_offsets, E + 1, "expert_offsets")
    if out is None:
        out = torch.empty((M_total, K), dtype=out_dtype, device=G.device)
    _room(out, M_total * K, "out", (torch.float32, torch.float16))
    _check(load().moe_nf4_grouped_gemm_t(_ptr(G), DT[G.dtype], G.shape[0], _ptr(packed),
                                         _ptr(absmax), _ptr(expert_offsets), E, N, K, M_total,
                                         _ptr(out), DT[out.dtype], ALGO[algo], _ptr(dev_err),
                                         _stream(G.device)), "moe_nf4_grouped_gemm_t")
    return out


def nf4_down_backward(dYp, packed, absmax, expert_offsets, M_total, gu, out_dtype=torch.float32,
                      out=None, dev_err=None):
    """Transposed down GEMM + SwiGLU backward in one tensor-core launch:
    ``dYp`` fp16 ``[>= M_total, H]``, the down stack ``[E, H, I]``, ``gu`` fp32
    ``[M_total, 2I]`` (the forward's pre-activations) -> ``dgu [M_total, 2I]``."""
    _need(dYp, torch.float16, "dYp", 2)
    _need(packed, torch.uint8, "packed", 3)
    _need(absmax, torch.float32, "absmax")
    _need(expert_offsets, torch.int32, "expert_offsets", 1)
    _need(gu, torch.float32, "gu", 2)
    E, H, half = packed.shape
    I = 2 * half
    if dYp.shape[1] != H or gu.shape[1] != 2 * I:
        raise MoEError("dYp [*, H] and gu [*, 2I] must match the down stack [E, H, I]")
    _room(absmax, E * H * (I // 64), "absmax")
    _room(expert_offsets, E + 1, "expert_offsets")
    _room(gu, M_total * 2 * I, "gu")
    if out is None:
        out = torch.empty((M_total, 2 * I), dtype=out_dtype, device=dYp.device)
    _room(out, M_total * 2 * I, "out", (torch.float32, torch.float16))
    _check(load().moe_nf4_down_backward(_ptr(dYp), dYp.shape[0], _ptr(packed), _ptr(absmax),
                                        _ptr(expert_offsets), E, H, I, M_total, _ptr(gu),
                                        _ptr(out), DT[out.dtype], _ptr(dev_err),
                                        _stream(dYp.device)), "moe_nf4_down_backward")
    return out


def swiglu_backward(gu, dh, out_dtype=torch.float32, out=None):
    """``gu [M, 2I]``, ``dh [M, I]`` (same dtype, fp32 or fp16) -> ``dgu [M, 2I]``."""
    _need(gu, gu.dtype, "gu", 2)
    _need(dh, gu.dtype, "dh", 2)
    M, two_i = gu.shape
    if dh.shape != (M, two_i // 2):
        raise MoEError("dh must be [M, I] for gu [M, 2I]")
    if out is None:
        out = torch.empty((M, two_i), dtype=out_dtype, device=gu.device)
    _room(out, M * two_i, "out", (torch.float32, torch.float16))
    _check(load().moe_swiglu_backward(_ptr(gu), _ptr(dh), DT[gu.dtype], M, two_i // 2, _ptr(out),
                                      DT[out.dtype], _stream(gu.device)), "moe_swiglu_backward")
    return out


def combine_backward(dY, Yp, inv_perm, topk_w, dyp_dtype=torch.float32, dev_err=None):
    """Adjoint of ``unpermute_combine``: ``(dYp [T*k, H], dw fp32 [T, k])``."""
    _need(dY, torch.float32, "dY", 2)
    _need(Yp, Yp.dtype, "Yp", 2)
    _need(inv_perm, torch.int32, "inv_perm")
    _need(topk_w, torch.float32, "topk_w", 2)
    T, k = topk_w.shape
    H = dY.shape[1]
    if dY.shape[0] != T:
        raise MoEError("dY must have one row per token of topk_w")
    _room(Yp, T * k * H, "Yp", (torch.float32, torch.float16))
    _room(inv_perm, T * k, "inv_perm")
    dYp = torch.empty((T * k, H), dtype=dyp_dtype, device=dY.device)
    dw = torch.empty((T, k), dtype=torch.float32, device=dY.device)
    _check(load().moe_combine_backward(_ptr(dY), _ptr(Yp), DT[Yp.dtype], _ptr(inv_perm),
                                       _ptr(topk_w), T, k, H, _ptr(dYp), DT[dYp.dtype], _ptr(dw),
                                       _ptr(dev_err), _stream(dY.device)), "moe_combine_backward")
    return dYp, dw


def route_backward(logits, topk_idx, topk_w, dw, renormalize, dev_err=None):
    """Gradient of the routing weights w.r.t. the logits -> ``fp32 [T, E]``."""
    _need(logits, torch.float32, "logits", 2)
    _need(topk_idx, torch.int32, "topk_idx", 2)
    _need(topk_w, torch.float32, "topk_w", 2)
    _need(dw, torch.float32, "dw", 2)
    T, E = logits.shape
    k = topk_idx.shape[1]
    for t, name in ((topk_idx, "topk_idx"), (topk_w, "topk_w"), (dw, "dw")):
        if tuple(t.shape) != (T, k):
            raise MoEError(f"{name} must be [T, k] = [{T}, {k}]")
    out = torch.empty((T, E), dtype=torch.float32, device=logits.device)
    _check(load().moe_route_backward(_ptr(logits), _ptr(topk_idx), _ptr(topk_w), _ptr(dw), T, E,
                                     k, int(bool(renormalize)), _ptr(out), _ptr(dev_err),
                                     _stream(logits.device)), "moe_route_backward")
    return out


def lora_delta(X, expert_offsets, lora_A, lora_B, scale, out, M_total=None, dev_err=None):
    """In place: ``out[p] += scale * lora_B[e(p)] @ (lora_A[e(p)] @ X[p])`` for
    the first ``M_total`` rows (default ``out``'s rows); ``X`` fp16 [>= M_total,
    K], ``lora_A`` fp16 [E, r, K], ``lora_B`` fp16 [E, N, r], ``out`` fp32 [M_total, N]."""
    _need(X, torch.float16, "X", 2)
    _need(expert_offsets, torch.int32, "expert_offsets", 1)
    _need(lora_A, torch.float16, "lora_A", 3)
    _need(lora_B, torch.float16, "lora_B", 3)
    _need(out, torch.float32, "out", 2)
    E, r, K = lora_A.shape
    N = lora_B.shape[1]
    if lora_B.shape != (E, N, r) or X.shape[1] != K or out.shape[1] != N:
        raise MoEError("lora_A [E, r, K], lora_B [E, N, r], X [*, K] and out [*, N] disagree")
    M = out.shape[0] if M_total is None else M_total
    if out.shape[0] < M:
        raise MoEError("out has fewer than M_total rows")
    _room(expert_offsets, E + 1, "expert_offsets")
    _check(load().moe_lora_delta(_ptr(X), X.shape[0], _ptr(expert_offsets), E, N, K, r,
                                 _ptr(lora_A), _ptr(lora_B), float(scale), M, _ptr(out),
                                 _ptr(dev_err), _stream(X.device)), "moe_lora_delta")
    return out


def permute_rows(X, sorted_rows, k, M_total=None, out=None, dev_err=None):
    """``Xp[p] = fp16(X[sorted_rows[p] // k])`` -> ``fp16 [M_total, K]``."""
    if X.dtype not in (torch.bfloat16, torch.float16):
        raise MoEError("X must be bf16 or fp16")
    _need(X, X.dtype, "X", 2)
    _need(sorted_rows, torch.int32, "sorted_rows", 1)
    T, K = X.shape
    M = sorted_rows.numel() if M_total is None else M_total
    _room(sorted_rows, M, "sorted_rows")
    if out is None:
        out = torch.empty((M, K), dtype=torch.float16, device=X.device)
    _room(out, M * K, "out", (torch.float16,))
    _check(load().moe_permute_rows(_ptr(X), DT[X.dtype], T, K, _ptr(sorted_rows), k, M,
                                   _ptr(out), _ptr(dev_err), _stream(X.device)),
           "moe_permute_rows")
    return out


def swiglu(gu, h_dtype=torch.float32, out=None):
    _need(gu, gu.dtype, "gu", 2)
    M, two_i = gu.shape
    if out is None:
        out = torch.empty((M, two_i // 2), dtype=h_dtype, device=gu.device)
    _room(out, M * (two_i // 2), "out", _F)
    _check(load().moe_swiglu(_ptr(gu), DT[gu.dtype], M, two_i // 2, _ptr(out), DT[out.dtype],
                             _stream(gu.device)), "moe_swiglu")
    return out


def unpermute_combine(Yp, inv_perm, topk_w, y_dtype=torch.float32, out=None):
    _need(Yp, Yp.dtype, "Yp", 2)
    _need(inv_perm, torch.int32, "inv_perm")
    _need(topk_w, torch.float32, "topk_w", 2)
    T, k = topk_w.shape
    H = Yp.shape[1]
    _room(Yp, T * k * H, "Yp", _F)
    _room(inv_perm, T * k, "inv_perm")
    if out is None:
        out = torch.empty((T, H), dtype=y_dtype, device=Yp.device)
    _room(out, T * H, "out", _F)
    _check(load().moe_unpermute_combine(_ptr(Yp), DT[Yp.dtype], _ptr(inv_perm), _ptr(topk_w),
                                        T, k, H, _ptr(out), DT[out.dtype], _stream(Yp.device)),
           "moe_unpermute_combine")
    return out


def layer_workspace_size(T, E, k, H, I):
    n = ctypes.c_size_t()
    _check(load().moe_layer_workspace_size(T, E, k, H, I, ctypes.byref(n)),
           "moe_layer_workspace_size")
    return n.value


def layer_forward(X, logits, k, renormalize, packed_gu, absmax_gu, packed_d, absmax_d,
                  workspace=None, out=None, dev_err=None):
    """The whole layer through one C call: ``Y fp32 [T, H]``."""
    _need(X, torch.bfloat16, "X", 2)
    _need(logits, torch.float32, "logits", 2)
    T, H = X.shape
    E = logits.shape[1]
    I = packed_d.shape[2] * 2
    if logits.shape[0] != T:
        raise MoEError("logits must have one row per token of X")
    _room(packed_gu, E * 2 * I * (H // 2), "packed_gu", (torch.uint8,))
    _room(absmax_gu, E * 2 * I * (H // 64), "absmax_gu", (torch.float32,))
    _room(packed_d, E * H * (I // 2), "packed_d", (torch.uint8,))
    _room(absmax_d, E * H * (I // 64), "absmax_d", (torch.float32,))
    nbytes = layer_workspace_size(T, E, k, H, I)
    if workspace is None:
        workspace = torch.empty((max(nbytes, 256),), dtype=torch.uint8, device=X.device)
    if out is None:
        out = torch.empty((T, H), dtype=torch.float32, device=X.device)
    _room(out, T * H, "out", (torch.float32,))
    _room(workspace, 0, "workspace")
    _check(load().moe_layer_forward(
        _ptr(X), _ptr(logits), T, E, k, 1 if renormalize else 0, H, I, _ptr(packed_gu),
        _ptr(absmax_gu), _ptr(packed_d), _ptr(absmax_d), _ptr(out), _ptr(workspace),
        workspace.numel(), _ptr(dev_err), _stream(X.device)), "moe_layer_forward")
    return out
