// C ABI of libmoenf4.so: argument validation and dispatch.  Every entry point
// checks its arguments on the host, then enqueues kernels on the caller's
// stream; nothing here synchronizes or allocates.
#include <cstdint>

#include "common.cuh"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status_t check_device() {
  moe::DeviceInfo d;
  if (!moe::device_info(&d)) return MOE_ERR_CUDA;
  return (d.major == 10 && d.minor == 0) ? MOE_OK : MOE_ERR_UNSUPPORTED;
}

// The CUDA error behind the calling thread's most recent MOE_ERR_CUDA.
thread_local cudaError_t t_last_cuda_error = cudaSuccess;

moe_status_t from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  t_last_cuda_error = e;
  return MOE_ERR_CUDA;
}

bool valid_dtype(moe_dtype_t d) { return d == MOE_DT_F32 || d == MOE_DT_BF16 || d == MOE_DT_F16; }
bool f32_or_f16(moe_dtype_t d) { return d == MOE_DT_F32 || d == MOE_DT_F16; }

size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

}  // namespace

extern "C" {

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_MISALIGNED: return "MOE_ERR_MISALIGNED";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
  }
  return "MOE_ERR_UNKNOWN";
}

int moe_abi_version(void) { return MOE_NF4_ABI_VERSION; }

const char* moe_last_cuda_error(void) {
  return t_last_cuda_error == cudaSuccess ? "no error" : cudaGetErrorString(t_last_cuda_error);
}

moe_status_t moe_nf4_levels(float* levels_out) {
  if (!levels_out) return MOE_ERR_INVALID_ARG;
  static const float kLevels[16] = {MOE_NF4_LEVEL_LIST};
  for (int i = 0; i < 16; ++i) levels_out[i] = kLevels[i];
  return MOE_OK;
}

moe_status_t moe_nf4_quantize(const float* W, int E, int N, int K, int blocksize,
                              uint8_t* packed, float* absmax, int32_t* dev_err, void* stream) {
  if (blocksize != moe::kBlock || E < 1 || N < 1 || K < 1 || K % moe::kBlock)
    return MOE_ERR_INVALID_ARG;
  if (!W || !packed || !absmax) return MOE_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(packed) || !aligned16(absmax)) return MOE_ERR_MISALIGNED;
  if (moe_status_t st = check_device()) return st;
  return from_cuda(moe_launch::nf4_quantize(W, (int64_t)E * N, K, packed, absmax, dev_err,
                                            (cudaStream_t)stream));
}

moe_status_t moe_int4_quantize(const float* W, int E, int N, int K, uint8_t* packed,
                               uint32_t* meta, int32_t* dev_err, void* stream) {
  if (E < 1 || N < 1 || K < 1 || K % 128) return MOE_ERR_INVALID_ARG;
  if (!W || !packed || !meta) return MOE_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(packed) || !aligned16(meta)) return MOE_ERR_MISALIGNED;
  if (moe_status_t st = check_device()) return st;
  return from_cuda(moe_launch::int4_quantize(W, (int64_t)E * N, K, packed, meta, dev_err,
                                             (cudaStream_t)stream));
}

moe_status_t moe_int4_grouped_gemm(const void* A, int A_rows, const uint8_t* packed,
                                   const uint32_t* meta, const int32_t* expert_offsets, int E,
                                   int N, int K, int M_total, moe_epilogue_t epilogue, void* out,
                                   moe_dtype_t out_dtype, moe_algo_t algo, int32_t* dev_err,
                                   void* stream) {
  if (E < 1 || E > 1024 || N < 1 || K < 1 || M_total < 0 || A_rows < M_total)
    return MOE_ERR_INVALID_ARG;
  if (epilogue != MOE_EPI_NONE && epilogue != MOE_EPI_SWIGLU) return MOE_ERR_INVALID_ARG;
  if (!valid_dtype(out_dtype)) return MOE_ERR_INVALID_ARG;
  if (algo != MOE_ALGO_AUTO && algo != MOE_ALGO_GEMV && algo != MOE_ALGO_TC)
    return MOE_ERR_INVALID_ARG;
  const bool gemv_ok = moe_launch::grouped_gemm_int4_supported(N, K);
  const bool tc_ok = moe_launch::grouped_gemm_tc_supported(N, K, epilogue) && K % 128 == 0;
  const bool use_tc = algo == MOE_ALGO_TC ||
                      (algo == MOE_ALGO_AUTO && tc_ok && ((int64_t)M_total >= 36LL * E || !gemv_ok));
  if (use_tc ? !tc_ok : !gemv_ok) return MOE_ERR_UNSUPPORTED;
  if (!expert_offsets || !packed || !meta) return MOE_ERR_INVALID_ARG;
  if (M_total > 0 && (!A || !out)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {A, packed, meta, expert_offsets, out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  if (moe_status_t st = check_device()) return st;
  if (M_total == 0) return MOE_OK;
  if (use_tc)
    return from_cuda(moe_launch::grouped_gemm_tc_int4(A, A_rows, packed, meta, expert_offsets, E,
                                                      N, K, M_total, epilogue, out, out_dtype,
                                                      dev_err, (cudaStream_t)stream));
  return from_cuda(moe_launch::grouped_gemm_int4(A, A_rows, packed, meta, expert_offsets, E, N,
                                                 K, M_total, epilogue, out, out_dtype, dev_err,
                                                 (cudaStream_t)stream));
}

moe_status_t moe_mxfp4_quantize(const float* W, int E, int N, int K, uint8_t* packed,
                                uint8_t* scales, int32_t* dev_err, void* stream) {
  if (E < 1 || N < 1 || K < 1 || K % 32) return MOE_ERR_INVALID_ARG;
  if (!W || !packed || !scales) return MOE_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(packed) || !aligned16(scales)) return MOE_ERR_MISALIGNED;
  if (moe_status_t st = check_device()) return st;
  return from_cuda(moe_launch::mxfp4_quantize(W, (int64_t)E * N, K, packed, scales, dev_err,
                                              (cudaStream_t)stream));
}

moe_status_t moe_mxfp4_grouped_gemm(const void* A, int A_rows, const uint8_t* packed,
                                    const uint8_t* scales, const int32_t* expert_offsets, int E,
                                    int N, int K, int M_total, moe_epilogue_t epilogue, void* out,
                                    moe_dtype_t out_dtype, moe_algo_t algo, int32_t* dev_err,
                                    void* stream) {
  if (E < 1 || E > 1024 || N < 1 || K < 1 || M_total < 0 || A_rows < M_total)
    return MOE_ERR_INVALID_ARG;
  if (epilogue != MOE_EPI_NONE && epilogue != MOE_EPI_SWIGLU) return MOE_ERR_INVALID_ARG;
  if (!valid_dtype(out_dtype)) return MOE_ERR_INVALID_ARG;
  if (algo != MOE_ALGO_AUTO && algo != MOE_ALGO_GEMV && algo != MOE_ALGO_TC &&
      algo != MOE_ALGO_TC_PAIR)
    return MOE_ERR_INVALID_ARG;
  const bool gemv_ok = moe_launch::grouped_gemm_mxfp4_supported(N, K);
  const bool pair = algo == MOE_ALGO_TC_PAIR;
  const bool tc_ok = moe_launch::grouped_gemm_tc_supported(N, K, epilogue) && (!pair || N % 256 == 0);
  bool use_tc;
  if (algo == MOE_ALGO_TC || pair) use_tc = true;
  else if (algo == MOE_ALGO_GEMV) use_tc = false;
  else use_tc = tc_ok && ((int64_t)M_total >= 36LL * E || !gemv_ok);  // the NF4 rule
  if (use_tc ? !tc_ok : !gemv_ok) return MOE_ERR_UNSUPPORTED;
  if (!expert_offsets || !packed || !scales) return MOE_ERR_INVALID_ARG;
  if (M_total > 0 && (!A || !out)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {A, packed, scales, expert_offsets, out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  if (moe_status_t st = check_device()) return st;
  if (M_total == 0) return MOE_OK;
  if (use_tc)
    return from_cuda(moe_launch::grouped_gemm_tc_mxfp4(A, A_rows, packed, scales, expert_offsets,
                                                       E, N, K, M_total, epilogue, out,
                                                       out_dtype, dev_err, (cudaStream_t)stream,
                                                       pair));
  return from_cuda(moe_launch::grouped_gemm_mxfp4(A, A_rows, packed, scales, expert_offsets, E, N,
                                                  K, M_total, epilogue, out, out_dtype, dev_err,
                                                  (cudaStream_t)stream));
}

moe_status_t moe_nf4_grouped_gemm_t(const void* G, moe_dtype_t g_dtype, int G_rows,
                                    const uint8_t* packed, const float* absmax,
                                    const int32_t* expert_offsets, int E, int N, int K,
                                    int M_total, void* out, moe_dtype_t out_dtype,
                                    moe_algo_t algo, int32_t* dev_err, void* stream) {
  if (!f32_or_f16(g_dtype) || !f32_or_f16(out_dtype)) return MOE_ERR_INVALID_ARG;
  if (algo != MOE_ALGO_AUTO && algo != MOE_ALGO_GEMV && algo != MOE_ALGO_TC)
    return MOE_ERR_INVALID_ARG;
  if (E < 1 || E > 1024 || N < 1 || K < 1 || K % moe::kBlock || M_total < 0 || G_rows < M_total)
    return MOE_ERR_INVALID_ARG;
  if (!expert_offsets || !packed || !absmax) return MOE_ERR_INVALID_ARG;
  if (M_total > 0 && (!G || !out)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {G, packed, absmax, expert_offsets, out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  const bool tc_ok = g_dtype == MOE_DT_F16 && moe_launch::grouped_gemm_t_tc_supported(N, K);
  if (algo == MOE_ALGO_TC && !tc_ok) return MOE_ERR_UNSUPPORTED;
  const bool use_tc =
      algo == MOE_ALGO_TC || (algo == MOE_ALGO_AUTO && tc_ok && (int64_t)M_total >= 36LL * E);
  if (moe_status_t st = check_device()) return st;
  if (use_tc) {
    if (M_total == 0) return MOE_OK;
    return from_cuda(moe_launch::grouped_gemm_t_tc(G, G_rows, packed, absmax, expert_offsets, E,
                                                   N, K, M_total, false, nullptr, out, out_dtype,
                                                   dev_err, (cudaStream_t)stream));
  }
  return from_cuda(moe_launch::grouped_gemm_t(G, g_dtype, packed, absmax, expert_offsets, E, N, K,
                                              M_total, out, out_dtype, dev_err,
                                              (cudaStream_t)stream));
}

moe_status_t moe_nf4_down_backward(const void* dYp, int G_rows, const uint8_t* packed,
                                   const float* absmax, const int32_t* expert_offsets, int E,
                                   int H, int I, int M_total, const float* gu, void* dgu,
                                   moe_dtype_t dgu_dtype, int32_t* dev_err, void* stream) {
  if (!f32_or_f16(dgu_dtype)) return MOE_ERR_INVALID_ARG;
  if (E < 1 || E > 1024 || H < 1 || I < 1 || M_total < 0 || G_rows < M_total)
    return MOE_ERR_INVALID_ARG;
  if (!moe_launch::grouped_gemm_t_tc_supported(H, I)) return MOE_ERR_UNSUPPORTED;
  if (!expert_offsets || !packed || !absmax) return MOE_ERR_INVALID_ARG;
  if (M_total > 0 && (!dYp || !gu || !dgu)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {dYp, packed, absmax, expert_offsets, gu, dgu};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  if (moe_status_t st = check_device()) return st;
  if (M_total == 0) return MOE_OK;
  return from_cuda(moe_launch::grouped_gemm_t_tc(dYp, G_rows, packed, absmax, expert_offsets, E, H,
                                                 I, M_total, true, gu, dgu, dgu_dtype, dev_err,
                                                 (cudaStream_t)stream));
}

moe_status_t moe_swiglu_backward(const void* gu, const void* dh, moe_dtype_t in_dtype, int M,
                                 int I, void* dgu, moe_dtype_t out_dtype, void* stream) {
  if (!f32_or_f16(in_dtype) || !f32_or_f16(out_dtype) || M < 0 || I < 1)
    return MOE_ERR_INVALID_ARG;
  if (M > 0 && (!gu || !dh || !dgu)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {gu, dh, dgu};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  if (moe_status_t st = check_device()) return st;
  return from_cuda(
      moe_launch::swiglu_backward(gu, dh, in_dtype, M, I, dgu, out_dtype, (cudaStream_t)stream));
}

moe_status_t moe_combine_backward(const float* dY, const void* Yp, moe_dtype_t yp_dtype,
                                  const int32_t* inv_perm, const float* topk_w, int T, int k,
                                  int H, void* dYp, moe_dtype_t dyp_dtype, float* dw,
                                  int32_t* dev_err, void* stream) {
  if (!f32_or_f16(yp_dtype) || !f32_or_f16(dyp_dtype) || T < 0 || k < 1 || k > 32 || H < 1)
    return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!dY || !Yp || !inv_perm || !topk_w || !dYp || !dw)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {dY, Yp, inv_perm, topk_w, dYp, dw};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  if (moe_status_t st = check_device()) return st;
  return from_cuda(moe_launch::combine_backward(dY, Yp, yp_dtype, inv_perm, topk_w, T, k, H, dYp,
                                                dyp_dtype, dw, dev_err, (cudaStream_t)stream));
}

moe_status_t moe_route_backward(const float* logits, const int32_t* topk_idx,
                                const float* topk_w, const float* dw, int T, int E, int k,
                                int renormalize, float* dlogits, int32_t* dev_err, void* stream) {
  if (T < 0 || E < 1 || E > 1024 || k < 1 || k > E || k > 32) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!logits || !topk_idx || !topk_w || !dw || !dlogits)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {logits, topk_idx, topk_w, dw, dlogits};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  if (moe_status_t st = check_device()) return st;
  return from_cuda(moe_launch::route_backward(logits, topk_idx, topk_w, dw, T, E, k, renormalize,
                                              dlogits, dev_err, (cudaStream_t)stream));
}

moe_status_t moe_lora_delta(const void* X, int A_rows, const int32_t* expert_offsets, int E,
                            int N, int K, int r, const void* lora_A, const void* lora_B,
                            float scale, int M_total, float* out, int32_t* dev_err,
                            void* stream) {
  if (E < 1 || N < 1 || K < 1 || r < 1 || M_total < 0 || A_rows < M_total)
    return MOE_ERR_INVALID_ARG;
  if (!moe_launch::lora_delta_supported(E, K, r)) return MOE_ERR_UNSUPPORTED;
  if (!expert_offsets || !lora_A || !lora_B) return MOE_ERR_INVALID_ARG;
  if (M_total > 0 && (!X || !out)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {X, expert_offsets, lora_A, lora_B, out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  if (moe_status_t st = check_device()) return st;
  if (M_total == 0) return MOE_OK;
  return from_cuda(moe_launch::lora_delta(X, expert_offsets, E, N, K, r, lora_A, lora_B, scale,
                                          M_total, out, dev_err, (cudaStream_t)stream));
}

moe_status_t moe_nf4_dequantize(const uint8_t* packed, const float* absmax, int E, int N, int K,
                                void* out, moe_dtype_t out_dtype, void* stream) {
  if (E < 1 || N < 1 || K < 1 || K % moe::kBlock || !valid_dtype(out_dtype))
    return MOE_ERR_INVALID_ARG;
  if (!packed || !absmax || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(absmax) || !aligned16(out)) return MOE_ERR_MISALIGNED;
  if (moe_status_t st = check_device()) return st;
  return from_cuda(moe_launch::nf4_dequantize(packed, absmax, (int64_t)E * N, K, out, out_dtype,
                                              (cudaStream_t)stream));
}

moe_status_t moe_route_permute_workspace_size(int T, int E, int k, size_t* bytes) {
  if (!bytes || T < 0 || E < 1 || E > 1024 || k < 1 || k > E || k > 32)
    return MOE_ERR_INVALID_ARG;
  *bytes = moe_launch::route_workspace_bytes(T, E, k);
  return MOE_OK;
}

moe_status_t moe_route_permute(const float* logits, int T, int E, int k, int renormalize,
                               int32_t* topk_idx, float* topk_w, int32_t* expert_offsets,
                               int32_t* sorted_rows, int32_t* inv_perm, void* workspace,
                               size_t workspace_bytes, void* stream) {
  if (T < 0 || E < 1 || E > 1024 || k < 1 || k > E || k > 32) return MOE_ERR_INVALID_ARG;
  if ((int64_t)T * k > INT32_MAX / 2) return MOE_ERR_UNSUPPORTED;
  if (!expert_offsets) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!logits || !topk_idx || !topk_w || !sorted_rows || !inv_perm || !workspace))
    return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {logits, topk_idx, topk_w, expert_offsets, sorted_rows, inv_perm,
                        workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  if (T > 0 && workspace_bytes < moe_launch::route_workspace_bytes(T, E, k))
    return MOE_ERR_WORKSPACE;
  if (moe_status_t st = check_device()) return st;
  return from_cuda(moe_launch::route_permute(logits, T, E, k, renormalize ? 1 : 0, topk_idx,
                                             topk_w, expert_offsets, sorted_rows, inv_perm,
                                             workspace, (cudaStream_t)stream));
}

moe_status_t moe_route_permute_noalloc(const float* logits, int T, int E, int k,
                                       int renormalize, int32_t* topk_idx, float* topk_w,
                                       int32_t* expert_offsets, int32_t* sorted_rows,
                                       int32_t* inv_perm, void* stream) {
  if (T < 0 || E < 1 || E > 1024 || k < 1 || k > E || k > 32) return MOE_ERR_INVALID_ARG;
  if (!expert_offsets) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!logits || !topk_idx || !topk_w || !sorted_rows || !inv_perm))
    return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {logits, topk_idx, topk_w, expert_offsets, sorted_rows, inv_perm};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  if (!moe_launch::route_noalloc_fits(T, E, k)) return MOE_ERR_WORKSPACE;
  if (moe_status_t st = check_device()) return st;
  return from_cuda(moe_launch::route_permute_noalloc(logits, T, E, k, renormalize ? 1 : 0,
                                                     topk_idx, topk_w, expert_offsets,
                                                     sorted_rows, inv_perm,
                                                     (cudaStream_t)stream));
}

}  // extern "C"

namespace {

// moe_nf4_grouped_gemm; chain = true only from moe_layer_forward, where the
// expert offsets were written two or more kernels before this one (see
// moe_launch::grouped_gemm_gemv).
moe_status_t nf4_grouped_gemm_impl(const void* A, moe_dtype_t a_dtype, int A_rows,
                                   const int32_t* gather, int k, const uint8_t* packed,
                                   const float* absmax, const int32_t* expert_offsets, int E,
                                   int N, int K, int M_total, moe_epilogue_t epilogue, void* out,
                                   moe_dtype_t out_dtype, moe_algo_t algo, int32_t* dev_err,
                                   void* stream, bool chain) {
  if (a_dtype != MOE_DT_BF16 && a_dtype != MOE_DT_F16) return MOE_ERR_INVALID_ARG;
  if (!valid_dtype(out_dtype)) return MOE_ERR_INVALID_ARG;
  if (epilogue != MOE_EPI_NONE && epilogue != MOE_EPI_SWIGLU) return MOE_ERR_INVALID_ARG;
  if (algo != MOE_ALGO_AUTO && algo != MOE_ALGO_GEMV && algo != MOE_ALGO_TC &&
      algo != MOE_ALGO_TC_PAIR)
    return MOE_ERR_INVALID_ARG;
  if (E < 1 || E > 1024 || N < 1 || K < 1 || M_total < 0 || A_rows < 0 || (gather && k < 1))
    return MOE_ERR_INVALID_ARG;
  if (!gather && A_rows < M_total) return MOE_ERR_INVALID_ARG;
  if (K % moe::kBlock || N % 64) return MOE_ERR_INVALID_ARG;
  if (!expert_offsets || !packed || !absmax) return MOE_ERR_INVALID_ARG;
  if (M_total > 0 && (!A || !out)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {A, gather, packed, absmax, expert_offsets, out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  if (moe_status_t st = check_device()) return st;
  if (M_total == 0) return MOE_OK;
  const cudaStream_t s = (cudaStream_t)stream;
  const bool tc_ok = moe_launch::grouped_gemm_tc_supported(N, K, epilogue) && !gather &&
                     a_dtype == MOE_DT_F16;
  const bool pair = algo == MOE_ALGO_TC_PAIR;
  bool use_tc;
  if (algo == MOE_ALGO_TC || pair) {
    if (!tc_ok || (pair && N % 256)) return MOE_ERR_UNSUPPORTED;
    use_tc = true;
  } else if (algo == MOE_ALGO_GEMV) {
    use_tc = false;
  } else {
    // The tensor-core kernel decodes every weight and issues every MMA
    // whatever the token count, so it only wins once experts average enough
    // rows to amortise that; on B200 both kernels take the same time at about
    // 36 rows per expert on the OLMoE and Qwen3 shapes (gate_up and down).
    use_tc = tc_ok && (int64_t)M_total >= 36LL * E;
  }
  if (use_tc)
    return from_cuda(moe_launch::grouped_gemm_tc(A, a_dtype, A_rows, gather, k, packed, absmax,
                                                 expert_offsets, E, N, K, M_total, epilogue,
                                                 out, out_dtype, dev_err, s, chain, pair));
  return from_cuda(moe_launch::grouped_gemm_gemv(A, a_dtype, A_rows, gather, k, packed, absmax,
                                                 expert_offsets, E, N, K, M_total, epilogue,
                                                 out, out_dtype, dev_err, s, chain));
}

}  // namespace

extern "C" {

moe_status_t moe_nf4_grouped_gemm(const void* A, moe_dtype_t a_dtype, int A_rows,
                                  const int32_t* gather, int k, const uint8_t* packed,
                                  const float* absmax, const int32_t* expert_offsets, int E,
                                  int N, int K, int M_total, moe_epilogue_t epilogue, void* out,
                                  moe_dtype_t out_dtype, moe_algo_t algo, int32_t* dev_err,
                                  void* stream) {
  return nf4_grouped_gemm_impl(A, a_dtype, A_rows, gather, k, packed, absmax, expert_offsets, E,
                               N, K, M_total, epilogue, out, out_dtype, algo, dev_err, stream,
                               false);
}

moe_status_t moe_permute_rows(const void* X, moe_dtype_t x_dtype, int T, int K,
                              const int32_t* sorted_rows, int k, int M_total, void* Xp,
                              int32_t* dev_err, void* stream) {
  if ((x_dtype != MOE_DT_BF16 && x_dtype != MOE_DT_F16) || T < 0 || K < 8 || K % 8 || k < 1 ||
      M_total < 0)
    return MOE_ERR_INVALID_ARG;
  if (M_total > 0 && (!X || !sorted_rows || !Xp)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {X, sorted_rows, Xp};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  if (moe_status_t st = check_device()) return st;
  return from_cuda(moe_launch::permute_rows(X, x_dtype, T, K, sorted_rows, k, M_total, Xp,
                                            dev_err, (cudaStream_t)stream));
}

moe_status_t moe_swiglu(const void* gu, moe_dtype_t gu_dtype, int M, int I, void* h,
                        moe_dtype_t h_dtype, void* stream) {
  if (!valid_dtype(gu_dtype) || !valid_dtype(h_dtype) || M < 0 || I < 1 || I % 4)
    return MOE_ERR_INVALID_ARG;
  if (M > 0 && (!gu || !h)) return MOE_ERR_INVALID_ARG;
  if ((gu && !aligned16(gu)) || (h && !aligned16(h))) return MOE_ERR_MISALIGNED;
  if (moe_status_t st = check_device()) return st;
  return from_cuda(moe_launch::swiglu(gu, gu_dtype, M, I, h, h_dtype, (cudaStream_t)stream));
}

moe_status_t moe_unpermute_combine(const void* Yp, moe_dtype_t yp_dtype, const int32_t* inv_perm,
                                   const float* topk_w, int T, int k, int H, void* Y,
                                   moe_dtype_t y_dtype, void* stream) {
  if (!valid_dtype(yp_dtype) || !valid_dtype(y_dtype) || T < 0 || k < 1 || k > 32 || H < 1 ||
      H % 4)
    return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!Yp || !inv_perm || !topk_w || !Y)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {Yp, inv_perm, topk_w, Y};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_MISALIGNED;
  if (moe_status_t st = check_device()) return st;
  return from_cuda(moe_launch::unpermute_combine(Yp, yp_dtype, inv_perm, topk_w, T, k, H, Y,
                                                 y_dtype, (cudaStream_t)stream));
}

// Layer workspace: [topk_idx | topk_w | offsets | sorted_rows | inv_perm |
// route scratch | Hbuf fp16 [T*k, I] | Yp fp16 [T*k, H] | Xp fp16 [T*k, H]],
// each 256-aligned.
static void layer_layout(int T, int E, int k, int H, int I, size_t off[9]) {
  const size_t tk = (size_t)T * k;
  off[0] = 0;
  off[1] = off[0] + align256(tk * 4);
  off[2] = off[1] + align256(tk * 4);
  off[3] = off[2] + align256((size_t)(E + 1) * 4);
  off[4] = off[3] + align256(tk * 4);
  off[5] = off[4] + align256(tk * 4);
  off[6] = off[5] + align256(moe_launch::route_workspace_bytes(T, E, k));
  off[7] = off[6] + align256(tk * I * 2);
  off[8] = off[7] + align256(tk * H * 2);
}

moe_status_t moe_layer_workspace_size(int T, int E, int k, int H, int I, size_t* bytes) {
  if (!bytes || T < 0 || E < 1 || E > 1024 || k < 1 || k > E || k > 32 || H < 1 || I < 1)
    return MOE_ERR_INVALID_ARG;
  size_t off[9];
  layer_layout(T, E, k, H, I, off);
  *bytes = off[8] + align256((size_t)T * k * H * 2);
  return MOE_OK;
}

moe_status_t moe_layer_forward(const void* X, const float* logits, int T, int E, int k,
                               int renormalize, int H, int I, const uint8_t* packed_gu,
                               const float* absmax_gu, const uint8_t* packed_d,
                               const float* absmax_d, float* Y, void* workspace,
                               size_t workspace_bytes, int32_t* dev_err, void* stream) {
  size_t need = 0;
  if (moe_status_t st = moe_layer_workspace_size(T, E, k, H, I, &need)) return st;
  if (T == 0) return MOE_OK;
  if (!workspace || workspace_bytes < need) return MOE_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MOE_ERR_MISALIGNED;
  size_t off[9];
  layer_layout(T, E, k, H, I, off);
  char* ws = reinterpret_cast<char*>(workspace);
  int32_t* topk_idx = reinterpret_cast<int32_t*>(ws + off[0]);
  float* topk_w = reinterpret_cast<float*>(ws + off[1]);
  int32_t* offsets = reinterpret_cast<int32_t*>(ws + off[2]);
  int32_t* sorted_rows = reinterpret_cast<int32_t*>(ws + off[3]);
  int32_t* inv_perm = reinterpret_cast<int32_t*>(ws + off[4]);
  void* rws = ws + off[5];
  void* hbuf = ws + off[6];
  void* yp = ws + off[7];
  const int M = T * k;
  moe_status_t st = moe_route_permute(logits, T, E, k, renormalize, topk_idx, topk_w, offsets,
                                      sorted_rows, inv_perm, rws, off[6] - off[5], stream);
  if (st) return st;
  // Routed activation rows in expert order, fp16: both grouped kernels read
  // them without a gather or a conversion in their inner loops.
  void* xp = ws + off[8];
  st = moe_permute_rows(X, MOE_DT_BF16, T, H, sorted_rows, k, M, xp, dev_err, stream);
  if (st) return st;
  // The GEMMs run in chain mode: the offsets come from the routing two and
  // three kernels back, so each GEMM starts streaming its weights while the
  // kernel before it finishes.
  st = nf4_grouped_gemm_impl(xp, MOE_DT_F16, M, nullptr, 1, packed_gu, absmax_gu, offsets, E,
                             2 * I, H, M, MOE_EPI_SWIGLU, hbuf, MOE_DT_F16, MOE_ALGO_AUTO,
                             dev_err, stream, true);
  if (st) return st;
  st = nf4_grouped_gemm_impl(hbuf, MOE_DT_F16, M, nullptr, 1, packed_d, absmax_d, offsets, E, H,
                             I, M, MOE_EPI_NONE, yp, MOE_DT_F16, MOE_ALGO_AUTO, dev_err, stream,
                             true);
  if (st) return st;
  return moe_unpermute_combine(yp, MOE_DT_F16, inv_perm, topk_w, T, k, H, Y, MOE_DT_F32, stream);
}

}  // extern "C"
