// Shared device helpers of the NF4 MoE library (sm_100a).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <string>
#include <type_traits>
#include <unordered_map>
#include <utility>

#include "../../include/moe_nf4.h"

namespace moe {

constexpr int kBlock = 64;  // NF4 block size along K

// The sixteen NF4 levels (fp32, ascending), as published with QLoRA's
// NormalFloat data type and shipped in the bitsandbytes layout the pages'
// kernel consumes unchanged ("grouped-nf4-gemm & experts-4bit", first and
// third bullets).  Code 7 is exactly 0; codes 0 and 15 are exactly -1, +1.
#define MOE_NF4_LEVEL_LIST                                                   \
  -1.0f, -0.6961928009986877f, -0.5250730514526367f, -0.39491748809814453f, \
      -0.28444138169288635f, -0.18477343022823334f, -0.09105003625154495f,  \
      0.0f, 0.07958029955625534f, 0.16093020141124725f,                     \
      0.24611230194568634f, 0.33791524171829224f, 0.44070982933044434f,     \
      0.5626170039176941f, 0.7229568362236023f, 1.0f

__device__ __forceinline__ void set_dev_err(int32_t* dev_err, int bits) {
  if (dev_err) atomicOr(reinterpret_cast<int*>(dev_err), bits);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Loads that bypass L1 allocation for streamed-once data (weights).
__device__ __forceinline__ uint2 ldg_stream_u2(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
               : "=r"(r.x), "=r"(r.y)
               : "l"(p));
  return r;
}
__device__ __forceinline__ uint4 ldg_stream_u4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Two bf16 (packed in a u32, element 0 in the low half) -> two fp16.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
  float lo = __uint_as_float(v << 16);
  float hi = __uint_as_float(v & 0xffff0000u);
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// True when storing v as OutT loses it: an fp16 store of a magnitude that
// rounds past 65504 (>= 65520) or of a NaN.  fp32 and bf16 stores hold every
// finite fp32 product of this library, so they never report.
template <typename OutT>
__device__ __forceinline__ bool overflows_out(float v) {
  if constexpr (std::is_same<OutT, __half>::value) return !(fabsf(v) < 65520.0f);
  else return false;
}

// out[i] = v rounded once to OutT; an fp16 overflow sets MOE_DEVERR_RANGE.
template <typename OutT>
__device__ __forceinline__ void store_checked(OutT* out, size_t i, float v, int32_t* dev_err) {
  if (overflows_out<OutT>(v)) set_dev_err(dev_err, MOE_DEVERR_RANGE);
  out[i] = from_f32<OutT>(v);
}

// Any of the eight fp16 values packed in a uint4 infinite or NaN.
__device__ __forceinline__ bool any_f16x8_nonfinite(uint4 o) {
  const uint32_t w[4] = {o.x, o.y, o.z, o.w};
  bool bad = false;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    bad |= ((w[i] & 0x7C00u) == 0x7C00u) || ((w[i] & 0x7C000000u) == 0x7C000000u);
  return bad;
}

// MXFP4 (OCP Microscaling v1.0) decoding shared by the MXFP4 GEMV and the
// tensor-core GEMM.
// fp16 bits of an E2M1 code's value: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6,
// bit 3 the sign.
__device__ __forceinline__ uint32_t e2m1_h(uint32_t c) {
  const uint32_t m = c & 7u;
  const uint32_t mag = m == 0 ? 0u : m == 1 ? 0x3800u : m == 2 ? 0x3C00u : m == 3 ? 0x3E00u
                     : m == 4 ? 0x4000u : m == 5 ? 0x4200u : m == 6 ? 0x4400u : 0x4600u;
  return mag | ((c & 8u) << 12);
}

// E8M0 byte -> {2^(b-127), 2^(b-127)} as fp16 bits, exact for b in [103, 142]
// (fp16 subnormals from 2^-24); 0 below.  `bad` is set when b is not 0 and
// the scaled E2M1 values would not all be exact in fp16 (b outside
// [104, 140]).
__device__ __forceinline__ uint32_t mx_scale_h2(uint32_t b, bool& bad) {
  bad |= (b != 0u) && (b < 104u || b > 140u);
  uint32_t h = 0;
  if (b >= 113u && b <= 142u) h = (b - 112u) << 10;   // normal: exponent field b - 127 + 15
  else if (b >= 103u && b < 113u) h = 1u << (b - 103u);  // subnormal: 2^-24 * 2^(b - 103)
  return h * 0x00010001u;
}

// Weight formats of the tensor-core GEMM.
enum WeightFormat { kFmtNF4 = 0, kFmtMXFP4 = 1, kFmtINT4 = 2 };

// silu(g) * u with silu(g) = g / (1 + exp(-g)), IEEE division.
__device__ __forceinline__ float swiglu_f32(float g, float u) {
  return __fdiv_rn(g, 1.0f + expf(-g)) * u;
}

// Programmatic dependent launch.  Every kernel of the layer is launched with
// programmatic stream serialization (launch_pdl below), so it may start
// while the kernel before it on the stream is still running.  Such a kernel
// calls pdl_wait() before it touches any memory the earlier kernel may read
// or write (pdl_wait returns once that kernel has completed and its writes
// are visible), and pdl_trigger() only after its own pdl_wait(), so at most
// two kernels of a stream ever overlap.  Launched without the attribute,
// pdl_wait() returns at once.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (no link-time dependency on libcuda).  Null if the driver lacks it.
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// A tensor map depends only on its arguments (address, sizes, strides, box,
// swizzle, promotion, fill), so each distinct map is encoded once and reused:
// a launch then costs a hash lookup instead of a driver call.  Same signature
// and results as cuTensorMapEncodeTiled.
inline CUresult encode_tiled_cached(CUtensorMap* out, CUtensorMapDataType dt, cuuint32_t rank,
                                    void* addr, const cuuint64_t* dims,
                                    const cuuint64_t* strides, const cuuint32_t* box,
                                    const cuuint32_t* estr, CUtensorMapInterleave il,
                                    CUtensorMapSwizzle sw, CUtensorMapL2promotion l2,
                                    CUtensorMapFloatOOBfill oob) {
  const auto enc = tensor_map_encoder();
  if (!enc || rank < 1 || rank > 5) return CUDA_ERROR_NOT_SUPPORTED;
  uint64_t key[24] = {};
  int n = 0;
  key[n++] = (uint64_t)dt;
  key[n++] = rank;
  key[n++] = (uint64_t)(uintptr_t)addr;
  for (cuuint32_t i = 0; i < rank; ++i) key[n++] = dims[i];
  for (cuuint32_t i = 0; i + 1 < rank; ++i) key[n++] = strides[i];
  for (cuuint32_t i = 0; i < rank; ++i) key[n++] = ((uint64_t)box[i] << 32) | estr[i];
  key[n++] = ((uint64_t)il << 48) | ((uint64_t)sw << 32) | ((uint64_t)l2 << 16) | (uint64_t)oob;
  const std::string k(reinterpret_cast<const char*>(key), n * sizeof(uint64_t));
  static std::mutex mu;
  static std::unordered_map<std::string, CUtensorMap> cache;
  {
    std::lock_guard<std::mutex> lock(mu);
    const auto it = cache.find(k);
    if (it != cache.end()) {
      *out = it->second;
      return CUDA_SUCCESS;
    }
  }
  const CUresult r = enc(out, dt, rank, addr, dims, strides, box, estr, il, sw, l2, oob);
  if (r == CUDA_SUCCESS) {
    std::lock_guard<std::mutex> lock(mu);
    if (cache.size() >= 4096) cache.clear();
    cache.emplace(k, *out);
  }
  return r;
}

// Compute capability and SM count of the current device, queried once per
// device.
struct DeviceInfo {
  int major, minor, sms;
};
inline bool device_info(DeviceInfo* out) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static DeviceInfo info[kMaxDevices];
  static bool known[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(mu);
  if (!known[dev]) {
    DeviceInfo d{};
    if (cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return false;
    info[dev] = d;
    known[dev] = true;
  }
  *out = info[dev];
  return true;
}
inline int device_sm_count() {
  DeviceInfo d;
  return device_info(&d) ? d.sms : 148;
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per kernel and device.
inline cudaError_t set_max_dynamic_smem_once(const void* kern, int bytes) {
  static std::mutex mu;
  static std::unordered_map<const void*, uint64_t> done;  // device bitmask
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const uint64_t bit = 1ull << (dev & 63);
  {
    std::lock_guard<std::mutex> lock(mu);
    const auto it = done.find(kern);
    if (it != done.end() && (it->second & bit)) return cudaSuccess;
  }
  err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (err == cudaSuccess) {
    std::lock_guard<std::mutex> lock(mu);
    done[kern] |= bit;
  }
  return err;
}

}  // namespace moe

// Host-side launchers implemented in the kernel files, called by api.cu.
namespace moe_launch {
cudaError_t nf4_quantize(const float* W, int64_t rows, int K, uint8_t* packed,
                         float* absmax, int32_t* dev_err, cudaStream_t s);
cudaError_t nf4_dequantize(const uint8_t* packed, const float* absmax,
                           int64_t rows, int K, void* out, moe_dtype_t dt,
                           cudaStream_t s);
size_t route_workspace_bytes(int T, int E, int k);
bool route_noalloc_fits(int T, int E, int k);
cudaError_t route_permute_noalloc(const float* logits, int T, int E, int k, int renorm,
                                  int32_t* topk_idx, float* topk_w, int32_t* offsets,
                                  int32_t* sorted_rows, int32_t* inv_perm, cudaStream_t s);
cudaError_t route_permute(const float* logits, int T, int E, int k, int renorm,
                          int32_t* topk_idx, float* topk_w, int32_t* offsets,
                          int32_t* sorted_rows, int32_t* inv_perm, void* ws,
                          cudaStream_t s);
// The grouped NF4 GEMMs.  chain = true only inside the library's own layer
// sequence (route -> permute_rows -> gate_up -> down), where expert_offsets
// were written at least two kernels earlier: the GEMM then reads them, and
// starts streaming weights, before the kernel right before it (which writes
// A) has finished.  chain = false waits for that kernel before any access.
cudaError_t grouped_gemm_gemv(const void* A, moe_dtype_t a_dt, int A_rows,
                              const int32_t* gather, int k,
                              const uint8_t* packed, const float* absmax,
                              const int32_t* offsets, int E, int N, int K,
                              int M_total, moe_epilogue_t epi, void* out,
                              moe_dtype_t out_dt, int32_t* dev_err,
                              cudaStream_t s, bool chain = false);
bool grouped_gemm_decode_supported(int N, int K);
cudaError_t grouped_gemm_decode(const void* A, int A_rows, const uint8_t* packed,
                                const float* absmax, const int32_t* offsets, int E, int N,
                                int K, int M_total, moe_epilogue_t epi, void* out,
                                moe_dtype_t out_dt, int32_t* dev_err, cudaStream_t s,
                                bool chain = false);
cudaError_t grouped_gemm_tc(const void* A, moe_dtype_t a_dt, int A_rows,
                            const int32_t* gather, int k,
                            const uint8_t* packed, const float* absmax,
                            const int32_t* offsets, int E, int N, int K,
                            int M_total, moe_epilogue_t epi, void* out,
                            moe_dtype_t out_dt, int32_t* dev_err,
                            cudaStream_t s, bool chain = false, bool pair = false);
bool grouped_gemm_tc_supported(int N, int K, moe_epilogue_t epi);
// The tensor-core kernel in its transposed form (the backward):
// out[p, k] = sum_n W[e(p)][n, k] G[p, n], G fp16 [G_rows, N]; with
// swiglu_bwd the result is the gradient of h and the epilogue writes the
// gradient of the gate_up pre-activations gu (fp32 [M_total, 2K]) into out
// [M_total, 2K].
bool grouped_gemm_t_tc_supported(int N, int K);
cudaError_t grouped_gemm_t_tc(const void* G, int G_rows, const uint8_t* packed,
                              const float* absmax, const int32_t* offsets, int E, int N, int K,
                              int M_total, bool swiglu_bwd, const float* gu, void* out,
                              moe_dtype_t out_dt, int32_t* dev_err, cudaStream_t s);
// The same tensor-core kernel on INT4 weights (meta uint32 [E, N, K/128]:
// fp16 scale | zero << 16); A fp16 rows in permuted order.
cudaError_t grouped_gemm_tc_int4(const void* A, int A_rows, const uint8_t* packed,
                                 const uint32_t* meta, const int32_t* offsets, int E, int N,
                                 int K, int M_total, moe_epilogue_t epi, void* out,
                                 moe_dtype_t out_dt, int32_t* dev_err, cudaStream_t s);
// The same tensor-core kernel on MXFP4 weights (scales uint8 [E, N, K/32]);
// A fp16 rows in permuted order.
cudaError_t grouped_gemm_tc_mxfp4(const void* A, int A_rows, const uint8_t* packed,
                                  const uint8_t* scales, const int32_t* offsets, int E, int N,
                                  int K, int M_total, moe_epilogue_t epi, void* out,
                                  moe_dtype_t out_dt, int32_t* dev_err, cudaStream_t s,
                                  bool pair = false);
cudaError_t int4_quantize(const float* W, int64_t rows, int K, uint8_t* packed, uint32_t* meta,
                          int32_t* dev_err, cudaStream_t s);
bool grouped_gemm_int4_supported(int N, int K);
cudaError_t grouped_gemm_int4(const void* A, int A_rows, const uint8_t* packed,
                              const uint32_t* meta, const int32_t* offsets, int E, int N, int K,
                              int M_total, moe_epilogue_t epi, void* out, moe_dtype_t out_dt,
                              int32_t* dev_err, cudaStream_t s);
cudaError_t mxfp4_quantize(const float* W, int64_t rows, int K, uint8_t* packed, uint8_t* scales,
                           int32_t* dev_err, cudaStream_t s);
bool grouped_gemm_mxfp4_supported(int N, int K);
cudaError_t grouped_gemm_mxfp4(const void* A, int A_rows, const uint8_t* packed,
                               const uint8_t* scales, const int32_t* offsets, int E, int N, int K,
                               int M_total, moe_epilogue_t epi, void* out, moe_dtype_t out_dt,
                               int32_t* dev_err, cudaStream_t s);
cudaError_t grouped_gemm_t(const void* G, moe_dtype_t g_dt, const uint8_t* packed,
                           const float* absmax, const int32_t* offsets, int E, int N, int K,
                           int M_total, void* out, moe_dtype_t out_dt, int32_t* dev_err,
                           cudaStream_t s);
cudaError_t swiglu_backward(const void* gu, const void* dh, moe_dtype_t in_dt, int M, int I,
                            void* dgu, moe_dtype_t out_dt, cudaStream_t s);
cudaError_t combine_backward(const float* dY, const void* Yp, moe_dtype_t yp_dt,
                             const int32_t* inv_perm, const float* topk_w, int T, int k, int H,
                             void* dYp, moe_dtype_t dyp_dt, float* dw, int32_t* dev_err,
                             cudaStream_t s);
cudaError_t route_backward(const float* logits, const int32_t* topk_idx, const float* topk_w,
                           const float* dw, int T, int E, int k, int renormalize, float* dlogits,
                           int32_t* dev_err, cudaStream_t s);
bool lora_delta_supported(int E, int K, int r);
cudaError_t lora_delta(const void* X, const int32_t* offsets, int E, int N, int K, int r,
                       const void* lora_A, const void* lora_B, float scale, int M_total,
                       float* out, int32_t* dev_err, cudaStream_t s);
cudaError_t permute_rows(const void* X, moe_dtype_t x_dt, int T, int K, const int32_t* rows,
                         int k, int M_total, void* Xp, int32_t* dev_err, cudaStream_t s);
cudaError_t swiglu(const void* gu, moe_dtype_t gu_dt, int M, int I, void* h,
                   moe_dtype_t h_dt, cudaStream_t s);
cudaError_t unpermute_combine(const void* Yp, moe_dtype_t yp_dt,
                              const int32_t* inv_perm, const float* topk_w,
                              int T, int k, int H, void* Y, moe_dtype_t y_dt,
                              cudaStream_t s);
}  // namespace moe_launch
