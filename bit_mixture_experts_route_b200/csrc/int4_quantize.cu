// Grouped INT4 quantization (the format of the INT4 decode GEMV).
//
// The pages' serving stack runs GPTQ-calibrated int4 experts ("Jordan
// Anderson", jordananderson-pages.pages.dev, section "grouped-nf4-gemm &
// experts-4bit", third bullet).  Per group of 128 consecutive elements of a
// row: lo = min(min x, 0), hi = max(max x, 0), s = fp16(fl32((hi - lo) / 15)),
// z = clamp(rint(-lo / s), 0, 15), q = clamp(rint(x / s) + z, 0, 15), with
// IEEE fp32 divisions and rint rounding half to even; a group whose stored
// scale is 0 gets z = 0 and q = 0.  Codes are round-to-nearest: GPTQ's
// calibration would choose others in the same format, and needs data.
// One warp per group, four elements per lane.
#include "common.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256) int4_quantize_kernel(const float4* __restrict__ W,
                                                            int64_t ngroups,
                                                            uint16_t* __restrict__ packed,
                                                            uint32_t* __restrict__ meta,
                                                            int32_t* dev_err) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t g = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); g < ngroups;
       g += warps) {
    const float4 v = W[g * 32 + lane];
    const float x[4] = {v.x, v.y, v.z, v.w};
    bool finite = true;
    float lo = x[0], hi = x[0];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      finite &= isfinite(x[i]);
      lo = fminf(lo, x[i]);
      hi = fmaxf(hi, x[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (!__all_sync(0xffffffffu, finite) && lane == 0) set_dev_err(dev_err, MOE_DEVERR_NONFINITE);
    lo = fminf(lo, 0.0f);
    hi = fmaxf(hi, 0.0f);
    const __half s16 = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
    const float s = __half2float(s16);
    uint32_t z = 0, q[4] = {0, 0, 0, 0};
    if (s != 0.0f) {
      z = (uint32_t)fminf(fmaxf(rintf(__fdiv_rn(-lo, s)), 0.0f), 15.0f);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        q[i] = (uint32_t)fminf(fmaxf(rintf(__fdiv_rn(x[i], s)) + (float)z, 0.0f), 15.0f);
    }
    // elements 4l .. 4l+3 -> bytes 2l, 2l+1, even element in the high nibble
    packed[g * 32 + lane] = (uint16_t)(((q[0] << 4) | q[1]) | (((q[2] << 4) | q[3]) << 8));
    if (lane == 0) meta[g] = (uint32_t)__half_as_ushort(s16) | (z << 16);
  }
}

}  // namespace
}  // namespace moe

namespace moe_launch {

cudaError_t int4_quantize(const float* W, int64_t rows, int K, uint8_t* packed, uint32_t* meta,
                          int32_t* dev_err, cudaStream_t s) {
  const int64_t ngroups = rows * (K / 128);
  if (ngroups == 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>((ngroups + 7) / 8, (int64_t)moe::device_sm_count() * 8);
  moe::int4_quantize_kernel<<<(int)blocks, 256, 0, s>>>(reinterpret_cast<const float4*>(W),
                                                        ngroups, reinterpret_cast<uint16_t*>(packed),
                                                        meta, dev_err);
  return cudaGetLastError();
}

}  // namespace moe_launch
