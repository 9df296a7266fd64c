// MXFP4 quantization (the format of the MXFP4 decode GEMV).
//
// OCP Microscaling v1.0 conversion, as the pages' MXFP4 path consumes it (e2m1
// elements, e8m0 scales: "MoE Training on Consumer GPUs", cerinamroth.com/ml,
// section "Task guides").  Per block of 32 consecutive elements of a row:
// shared = clamp(floor(log2 max|x|) - 2, -127, 127), scale byte shared + 127;
// each y = x * 2^-shared (exact, fp32) becomes the nearest E2M1 value, ties to
// the even mantissa, magnitudes above 6 saturating to 6; a value that rounds
// to zero gets code 0; an all-zero block gets scale byte 0 and codes 0.
// Codes pack two per byte with element 2j in the low nibble.
// One warp covers four blocks (128 elements), four elements per lane.
#include "common.cuh"

namespace moe {
namespace {

// E2M1 code of |y| <= 6 (after saturation): the count of midpoints below it,
// where a value equal to a midpoint goes to the neighbour with an even
// mantissa bit (codes 0, 2, 4, 6).
__device__ __forceinline__ uint32_t e2m1_code(float y) {
  const float a = fminf(fabsf(y), 6.0f);
  uint32_t c = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) +
               (a >= 3.5f) + (a > 5.0f);
  if (c != 0u && signbit(y)) c |= 8u;
  return c;
}

// floor(log2 a) of a finite a > 0, from its bits (subnormals included)
__device__ __forceinline__ int floor_log2(float a) {
  const uint32_t bits = __float_as_uint(a);
  const int e = (int)((bits >> 23) & 0xFFu);
  if (e != 0) return e - 127;
  return (31 - __clz((int)(bits & 0x7FFFFFu))) - 149;
}

__global__ void __launch_bounds__(256) mxfp4_quantize_kernel(const float4* __restrict__ W,
                                                             int64_t nblocks,
                                                             uint16_t* __restrict__ packed,
                                                             uint8_t* __restrict__ scales,
                                                             int32_t* dev_err) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t nquads = (nblocks + 3) / 4;
  for (int64_t q = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); q < nquads;
       q += warps) {
    // lanes 8i .. 8i+7 hold block 4q + i, elements 4 (lane & 7) .. + 3
    const int64_t blk = 4 * q + (lane >> 3);
    const bool live = blk < nblocks;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (live) v = W[blk * 8 + (lane & 7)];
    const float x[4] = {v.x, v.y, v.z, v.w};
    bool finite = true;
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      finite &= isfinite(x[i]);
      amax = fmaxf(amax, fabsf(x[i]));
    }
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (!__all_sync(0xffffffffu, finite) && lane == 0) set_dev_err(dev_err, MOE_DEVERR_NONFINITE);
    uint32_t c[4] = {0u, 0u, 0u, 0u};
    uint32_t sbyte = 0u;
    if (amax > 0.0f) {
      const int shared = min(max(floor_log2(amax) - 2, -127), 127);
      // 2^-shared as an fp32 (biased exponent 127 - shared lies in [1, 254]
      // because floor_log2 of a finite fp32 is at most 127)
      const float inv = __uint_as_float((uint32_t)(127 - shared) << 23);
#pragma unroll
      for (int i = 0; i < 4; ++i) c[i] = e2m1_code(__fmul_rn(x[i], inv));
      sbyte = (uint32_t)(shared + 127);
    }
    if (live) {
      // elements 4l .. 4l+3 of the block -> bytes 2l (elements 4l, 4l+1) and
      // 2l+1 (4l+2, 4l+3), even element in the low nibble
      packed[blk * 8 + (lane & 7)] =
          (uint16_t)((c[0] | (c[1] << 4)) | ((c[2] | (c[3] << 4)) << 8));
      if ((lane & 7) == 0) scales[blk] = (uint8_t)sbyte;
    }
  }
}

}  // namespace
}  // namespace moe

namespace moe_launch {

cudaError_t mxfp4_quantize(const float* W, int64_t rows, int K, uint8_t* packed, uint8_t* scales,
                           int32_t* dev_err, cudaStream_t s) {
  const int64_t nblocks = rows * (K / 32);
  if (nblocks == 0) return cudaSuccess;
  const int64_t nquads = (nblocks + 3) / 4;
  const int64_t blocks = std::min<int64_t>((nquads + 7) / 8, (int64_t)moe::device_sm_count() * 8);
  moe::mxfp4_quantize_kernel<<<(int)blocks, 256, 0, s>>>(reinterpret_cast<const float4*>(W),
                                                         nblocks,
                                                         reinterpret_cast<uint16_t*>(packed),
                                                         scales, dev_err);
  return cudaGetLastError();
}

}  // namespace moe_launch

