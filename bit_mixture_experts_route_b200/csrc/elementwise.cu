// Standalone SwiGLU and the routing-weighted unpermute/combine.
//
// Both are HBM-bound streaming kernels with 16-byte vector accesses.
//   swiglu:  h[m, i] = silu(gu[m, i]) * gu[m, I + i]
//   combine: Y[t, :] = sum_{j<k} w[t, j] * Yp[inv_perm[t*k + j], :], summed in
//            j order in fp32 (deterministic).
#include <type_traits>

#include "common.cuh"

namespace moe {
namespace {

template <typename T>
struct Vec4 {
  T v[4];
};

template <typename T>
__device__ __forceinline__ void load4(const T* p, float (&f)[4]) {
  if constexpr (sizeof(T) == 4) {
    const float4 u = *reinterpret_cast<const float4*>(p);
    f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
  } else {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const T* h = reinterpret_cast<const T*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = to_f32<T>(h[i]);
  }
}

template <typename T>
__device__ __forceinline__ void store4(T* p, const float (&f)[4]) {
  if constexpr (sizeof(T) == 4) {
    *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  } else {
    Vec4<T> o;
#pragma unroll
    for (int i = 0; i < 4; ++i) o.v[i] = from_f32<T>(f[i]);
    *reinterpret_cast<Vec4<T>*>(p) = o;
  }
}

template <typename InT, typename OutT>
__global__ void __launch_bounds__(256) swiglu_kernel(const InT* __restrict__ gu, int M, int I,
                                                     OutT* __restrict__ h) {
  pdl_wait();
  pdl_trigger();
  const int64_t per_row = I / 4;
  const int64_t total = (int64_t)M * per_row;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < total; q += stride) {
    const int64_t m = q / per_row, c = (q % per_row) * 4;
    float g[4], u[4], o[4];
    load4(gu + m * 2 * I + c, g);
    load4(gu + m * 2 * I + I + c, u);
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = swiglu_f32(g[i], u[i]);
    store4(h + m * I + c, o);
  }
}

template <typename InT, typename OutT>
__global__ void __launch_bounds__(256) combine_kernel(const InT* __restrict__ Yp,
                                                      const int32_t* __restrict__ inv_perm,
                                                      const float* __restrict__ w, int T,
                                                      int k, int H, OutT* __restrict__ Y) {
  // One CTA-row of threads per token; each thread owns 4 consecutive columns.
  // The k positions and weights are staged in shared memory first, so the k
  // row loads of a thread are independent and issue back to back.
  __shared__ int s_p[32];
  __shared__ float s_w[32];
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  if (t >= T) return;
  const int total = T * k;
  if (threadIdx.x < k) {
    const int p = inv_perm[(size_t)t * k + threadIdx.x];
    s_p[threadIdx.x] = (p >= 0 && p < total) ? p : -1;
    s_w[threadIdx.x] = w[(size_t)t * k + threadIdx.x];
  }
  __syncthreads();
  for (int c = (blockIdx.y * blockDim.x + threadIdx.x) * 4; c < H; c += gridDim.y * blockDim.x * 4) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
    for (int j = 0; j < k; ++j) {
      const int p = s_p[j];
      if (p < 0) continue;
      float y[4];
      load4(Yp + (size_t)p * H + c, y);
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = fmaf(s_w[j], y[i], acc[i]);
    }
    store4(Y + (size_t)t * H + c, acc);
  }
}

// Xp[p, :] = X[sorted_rows[p] / k, :] converted to fp16, one warp per row,
// 16-byte accesses.  Rows whose id is out of range are zero-filled and flagged.
// A bf16 value beyond fp16's range becomes inf in Xp and sets
// MOE_DEVERR_RANGE.
template <typename InT>
__global__ void __launch_bounds__(256) permute_rows_kernel(const InT* __restrict__ X, int T, int K,
                                                           const int32_t* __restrict__ rows, int k,
                                                           int M_total, __half* __restrict__ Xp,
                                                           int32_t* dev_err) {
  pdl_wait();
  pdl_trigger();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  bool ovf = false;
  for (int p = warp; p < M_total; p += nwarps) {
    const int f = rows[p];
    const bool ok = f >= 0 && f < M_total && f / k < T;
    if (!ok && lane == 0) set_dev_err(dev_err, MOE_DEVERR_BAD_INDEX);
    const InT* src = X + (size_t)(ok ? f / k : 0) * K;
    __half* dst = Xp + (size_t)p * K;
    // eight 16-byte loads in flight per lane before the first store: a row
    // costs about one memory latency even when the grid is a single CTA
    for (int c0 = lane * 8; c0 < K; c0 += 8 * 256) {
      uint4 u[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = c0 + i * 256;
        u[i] = (ok && c < K) ? *reinterpret_cast<const uint4*>(src + c) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = c0 + i * 256;
        if (c >= K) break;
        uint4 o = u[i];
        if constexpr (sizeof(InT) == 2 && !std::is_same<InT, __half>::value) {
          o = make_uint4(bf16x2_to_f16x2(o.x), bf16x2_to_f16x2(o.y), bf16x2_to_f16x2(o.z),
                         bf16x2_to_f16x2(o.w));
          ovf |= any_f16x8_nonfinite(o);
        }
        *reinterpret_cast<uint4*>(dst + c) = o;
      }
    }
  }
  // every lane of the warp leaves the row loop together (warp-uniform p)
  if (__any_sync(0xffffffffu, ovf) && lane == 0) set_dev_err(dev_err, MOE_DEVERR_RANGE);
}

int sm_count() { return device_sm_count(); }

template <typename InT>
cudaError_t swiglu_out(const InT* gu, int M, int I, void* h, moe_dtype_t h_dt, cudaStream_t s) {
  const int64_t total = (int64_t)M * (I / 4);
  int grid = (int)std::min<int64_t>((total + 255) / 256, (int64_t)sm_count() * 8);
  if (grid < 1) grid = 1;
  if (h_dt == MOE_DT_F32)
    return launch_pdl(swiglu_kernel<InT, float>, dim3(grid), dim3(256), 0, s, gu, M, I, (float*)h);
  if (h_dt == MOE_DT_F16)
    return launch_pdl(swiglu_kernel<InT, __half>, dim3(grid), dim3(256), 0, s, gu, M, I,
                      (__half*)h);
  return launch_pdl(swiglu_kernel<InT, __nv_bfloat16>, dim3(grid), dim3(256), 0, s, gu, M, I,
                    (__nv_bfloat16*)h);
}

template <typename InT>
cudaError_t combine_out(const InT* Yp, const int32_t* inv_perm, const float* w, int T, int k,
                        int H, void* Y, moe_dtype_t y_dt, cudaStream_t s) {
  const int threads = 256;
  const int ychunks = std::max(1, std::min((H / 4 + threads - 1) / threads, 8));
  const dim3 grid(T, ychunks);
  if (y_dt == MOE_DT_F32)
    return launch_pdl(combine_kernel<InT, float>, grid, dim3(threads), 0, s, Yp, inv_perm, w, T,
                      k, H, (float*)Y);
  if (y_dt == MOE_DT_F16)
    return launch_pdl(combine_kernel<InT, __half>, grid, dim3(threads), 0, s, Yp, inv_perm, w, T,
                      k, H, (__half*)Y);
  return launch_pdl(combine_kernel<InT, __nv_bfloat16>, grid, dim3(threads), 0, s, Yp, inv_perm,
                    w, T, k, H, (__nv_bfloat16*)Y);
}

}  // namespace
}  // namespace moe

namespace moe_launch {

cudaError_t permute_rows(const void* X, moe_dtype_t x_dt, int T, int K, const int32_t* rows,
                         int k, int M_total, void* Xp, int32_t* dev_err, cudaStream_t s) {
  if (M_total == 0) return cudaSuccess;
  const int grid = (int)std::min<int64_t>(((int64_t)M_total + 7) / 8,
                                          (int64_t)moe::sm_count() * 16);
  if (x_dt == MOE_DT_BF16)
    return moe::launch_pdl(moe::permute_rows_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, s,
                           (const __nv_bfloat16*)X, T, K, rows, k, M_total, (__half*)Xp,
                           dev_err);
  return moe::launch_pdl(moe::permute_rows_kernel<__half>, dim3(grid), dim3(256), 0, s,
                         (const __half*)X, T, K, rows, k, M_total, (__half*)Xp, dev_err);
}

cudaError_t swiglu(const void* gu, moe_dtype_t gu_dt, int M, int I, void* h, moe_dtype_t h_dt,
                   cudaStream_t s) {
  if (M == 0) return cudaSuccess;
  if (gu_dt == MOE_DT_F32) return moe::swiglu_out((const float*)gu, M, I, h, h_dt, s);
  if (gu_dt == MOE_DT_F16) return moe::swiglu_out((const __half*)gu, M, I, h, h_dt, s);
  return moe::swiglu_out((const __nv_bfloat16*)gu, M, I, h, h_dt, s);
}

cudaError_t unpermute_combine(const void* Yp, moe_dtype_t yp_dt, const int32_t* inv_perm,
                              const float* topk_w, int T, int k, int H, void* Y,
                              moe_dtype_t y_dt, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if (yp_dt == MOE_DT_F32)
    return moe::combine_out((const float*)Yp, inv_perm, topk_w, T, k, H, Y, y_dt, s);
  if (yp_dt == MOE_DT_F16)
    return moe::combine_out((const __half*)Yp, inv_perm, topk_w, T, k, H, Y, y_dt, s);
  return moe::combine_out((const __nv_bfloat16*)Yp, inv_perm, topk_w, T, k, H, Y, y_dt, s);
}

}  // namespace moe_launch
