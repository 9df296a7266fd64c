// NF4 blockwise quantization of a fused expert stack, and its inverse.
//
// "4-bit Mixture-of-Experts fine-tuning on small GPUs" (jordananderson.work),
// second bullet: the quantizer of the fused 3-D expert parameter; "grouped-
// nf4-gemm & experts-4bit" (jordananderson-pages.pages.dev), first bullet:
// the bitsandbytes packed layout, two codes per byte.  Block size 64, fp32
// absmax, element 2j in the high nibble.
//
// Work split: 8 consecutive threads own one 64-element block, 8 elements
// each (two 16-byte loads), so a warp covers 4 blocks = 1 KB of fp32 input
// with fully coalesced 128-bit loads and writes 4 x 32 packed bytes with
// 32-bit stores.  HBM-bound: 256 B read + 36 B written per block.
#include "common.cuh"

namespace moe {
namespace {

__constant__ float c_levels[16] = {MOE_NF4_LEVEL_LIST};

// code = #{i : n > M_i}, M_i = fl32(L_i + L_{i+1}) * 0.5, found by a
// branch-free binary search over the 15 sorted thresholds (padded with +inf).
__device__ __forceinline__ uint32_t nf4_code(float n, const float* M) {
  uint32_t c = 0;
  c += (n > M[c + 7]) ? 8u : 0u;
  c += (n > M[c + 3]) ? 4u : 0u;
  c += (n > M[c + 1]) ? 2u : 0u;
  c += (n > M[c + 0]) ? 1u : 0u;
  return c;
}

__global__ void __launch_bounds__(256) nf4_quantize_kernel(
    const float4* __restrict__ W, int64_t nblocks, uint32_t* __restrict__ packed,
    float* __restrict__ absmax, int32_t* dev_err) {
  __shared__ float M[16];
  if (threadIdx.x < 16) {
    const int i = threadIdx.x;
    M[i] = (i < 15) ? __fmul_rn(__fadd_rn(c_levels[i], c_levels[i + 1]), 0.5f)
                    : __int_as_float(0x7f800000);  // +inf sentinel
  }
  __syncthreads();

  const int64_t nthreads = nblocks * 8;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < nthreads;
       g += stride) {
    // The 8 lanes of a block have consecutive g and nthreads is a multiple
    // of 8, so a block's lanes are always in or out of the loop together and
    // the 8-lane shuffles below see the whole block.
    const float4 a = W[2 * g];
    const float4 b = W[2 * g + 1];
    float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    float m = 0.0f;
    bool finite = true;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      m = fmaxf(m, fabsf(x[i]));
      finite &= isfinite(x[i]);
    }
    const unsigned grp = 0xffu << (threadIdx.x & 24);
    m = fmaxf(m, __shfl_xor_sync(grp, m, 1));
    m = fmaxf(m, __shfl_xor_sync(grp, m, 2));
    m = fmaxf(m, __shfl_xor_sync(grp, m, 4));
    if (!finite) set_dev_err(dev_err, MOE_DEVERR_NONFINITE);

    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t c = 7u;
      if (m > 0.0f) c = nf4_code(__fdiv_rn(x[i], m), M);
      // byte j (little-endian position j) = (code[2j] << 4) | code[2j+1]
      word |= c << ((i >> 1) * 8 + ((i & 1) ? 0 : 4));
    }
    packed[g] = word;
    if ((g & 7) == 0) absmax[g >> 3] = m;
  }
}

template <typename T>
__device__ __forceinline__ T from_f64(double v);
template <>
__device__ __forceinline__ float from_f64<float>(double v) { return __double2float_rn(v); }
template <>
__device__ __forceinline__ __half from_f64<__half>(double v) { return __double2half(v); }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f64<__nv_bfloat16>(double v) {
  return __double2bfloat16(v);
}

template <typename OutT>
__global__ void __launch_bounds__(256) nf4_dequantize_kernel(
    const uint32_t* __restrict__ packed, const float* __restrict__ absmax,
    int64_t nwords, OutT* __restrict__ out) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < nwords; g += stride) {
    const uint32_t w = packed[g];
    const float a = absmax[g >> 3];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t c = (w >> ((i >> 1) * 8 + ((i & 1) ? 0 : 4))) & 15u;
      // The product of two fp32 values is exact in fp64; round it once.
      out[g * 8 + i] = from_f64<OutT>((double)c_levels[c] * (double)a);
    }
  }
}

int grid_for(int64_t threads) {
  const int sms = device_sm_count();
  int64_t blocks = (threads + 255) / 256;
  const int64_t cap = (int64_t)sms * 8;
  return (int)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

}  // namespace
}  // namespace moe

namespace moe_launch {

cudaError_t nf4_quantize(const float* W, int64_t rows, int K, uint8_t* packed,
                         float* absmax, int32_t* dev_err, cudaStream_t s) {
  const int64_t nblocks = rows * (K / moe::kBlock);
  if (nblocks == 0) return cudaSuccess;
  moe::nf4_quantize_kernel<<<moe::grid_for(nblocks * 8), 256, 0, s>>>(
      reinterpret_cast<const float4*>(W), nblocks,
      reinterpret_cast<uint32_t*>(packed), absmax, dev_err);
  return cudaGetLastError();
}

cudaError_t nf4_dequantize(const uint8_t* packed, const float* absmax,
                           int64_t rows, int K, void* out, moe_dtype_t dt,
                           cudaStream_t s) {
  const int64_t nwords = rows * (K / 8);
  if (nwords == 0) return cudaSuccess;
  const int grid = moe::grid_for(nwords);
  const uint32_t* p = reinterpret_cast<const uint32_t*>(packed);
  if (dt == MOE_DT_F32)
    moe::nf4_dequantize_kernel<float><<<grid, 256, 0, s>>>(p, absmax, nwords, (float*)out);
  else if (dt == MOE_DT_F16)
    moe::nf4_dequantize_kernel<__half><<<grid, 256, 0, s>>>(p, absmax, nwords, (__half*)out);
  else
    moe::nf4_dequantize_kernel<__nv_bfloat16>
        <<<grid, 256, 0, s>>>(p, absmax, nwords, (__nv_bfloat16*)out);
  return cudaGetLastError();
}

}  // namespace moe_launch
