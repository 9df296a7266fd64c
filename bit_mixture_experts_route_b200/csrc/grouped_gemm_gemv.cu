// Grouped NF4 GEMM, decode path, general-shape kernel (few routed rows per
// expert; HBM-bound).  Permuted fp16 activations with K % 256 == 0 go to the
// TMA-staged kernel in grouped_gemm_decode.cu; this one covers the rest
// (gathered or bf16 activations, other K) with direct loads.
//
// "grouped-nf4-gemm & experts-4bit" (jordananderson-pages.pages.dev), first
// bullet: one launch for all active experts, the 16-entry codebook decoded in
// registers, no dequantized weight copy in memory.  At decode sizes the work
// is streaming the NF4 bytes of every expert that received a token, so this
// kernel is measured against HBM bandwidth.
//
// Design (swap-AB): the weights are the M side of mma.sync.m16n8k16 (16
// weight rows per warp), the routed tokens the N side (8 per MMA).  Per
// 64-element block each lane loads 8 packed bytes of two rows, turns each
// byte into an fp16 pair with one shared-memory lookup (a byte -> {L[hi],
// L[lo]} table replicated per lane, so lookups never conflict), and feeds
// four MMAs whose K order is permuted so every lane's bytes are contiguous;
// the activations are loaded in the same permuted order.  The four MMAs of a
// block accumulate the unscaled level sums, which are then scaled by the
// block's fp32 absmax and added to the fp32 accumulator -- so the only
// rounding on the weight side is that of the 16 levels to fp16.
//
// CTA = 4 warps = 64 weight rows of one expert; grid = (N/64, E).  CTAs of
// experts with no rows exit at once.  With the SwiGLU epilogue a warp's 16
// rows are 8 gate rows and the 8 matching up rows, so silu(g)*u is formed in
// registers.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kWarps = 4;
constexpr int kRowsPerCta = 16 * kWarps;
constexpr int kUnroll = 8;  // 64-blocks of weights in flight per lane

__constant__ float c_levels_gemv[16] = {MOE_NF4_LEVEL_LIST};

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4],
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
      "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 16 activations x[r][kb .. kb+16) as 8 fp16 pairs.
template <typename AT>
__device__ __forceinline__ void load_x16(const AT* __restrict__ A, size_t off, uint32_t (&xf)[8]);
template <>
__device__ __forceinline__ void load_x16<__half>(const __half* __restrict__ A, size_t off,
                                                 uint32_t (&xf)[8]) {
  const uint4* p = reinterpret_cast<const uint4*>(A + off);
  const uint4 u = __ldg(p), v = __ldg(p + 1);
  xf[0] = u.x; xf[1] = u.y; xf[2] = u.z; xf[3] = u.w;
  xf[4] = v.x; xf[5] = v.y; xf[6] = v.z; xf[7] = v.w;
}
template <>
__device__ __forceinline__ void load_x16<__nv_bfloat16>(const __nv_bfloat16* __restrict__ A,
                                                        size_t off, uint32_t (&xf)[8]) {
  const uint4* p = reinterpret_cast<const uint4*>(A + off);
  const uint4 u = __ldg(p), v = __ldg(p + 1);
  xf[0] = bf16x2_to_f16x2(u.x); xf[1] = bf16x2_to_f16x2(u.y);
  xf[2] = bf16x2_to_f16x2(u.z); xf[3] = bf16x2_to_f16x2(u.w);
  xf[4] = bf16x2_to_f16x2(v.x); xf[5] = bf16x2_to_f16x2(v.y);
  xf[6] = bf16x2_to_f16x2(v.z); xf[7] = bf16x2_to_f16x2(v.w);
}



// Process one chunk of up to 8*NT8 tokens of expert e for this warp's rows.
template <typename AT, int EPI, typename OutT, int NT8>
__device__ __forceinline__ void gemv_chunk(
    const AT* __restrict__ A, int A_rows, const int32_t* __restrict__ gather, int k,
    const uint8_t* __restrict__ wrowA, const uint8_t* __restrict__ wrowB,
    const float* __restrict__ arowA, const float* __restrict__ arowB,
    const uint32_t* __restrict__ lut, int K, int N, int M_total, int p0, int cnt,
    int outColA, int outColB, OutT* __restrict__ out, int32_t* dev_err) {
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;

  // Activation rows of this lane's tokens (8j + g) and their validity.
  size_t xrow[NT8];
  bool xok[NT8];
#pragma unroll
  for (int j = 0; j < NT8; ++j) {
    const int tok = 8 * j + g;
    xok[j] = tok < cnt;
    size_t r = 0;
    if (xok[j]) {
      const int p = p0 + tok;
      if (gather) {
        const int f = gather[p];
        if (f < 0 || f >= M_total || f / k >= A_rows) {
          set_dev_err(dev_err, MOE_DEVERR_BAD_INDEX);
          xok[j] = false;
        } else {
          r = (size_t)(f / k);
        }
      } else {
        r = (size_t)p;
      }
    }
    xrow[j] = r * (size_t)K;
  }

  float acc[NT8][4];
#pragma unroll
  for (int j = 0; j < NT8; ++j)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[j][q] = 0.0f;

  const int nblk = K / kBlock;
  for (int b0 = 0; b0 < nblk; b0 += kUnroll) {
    uint2 wa[kUnroll], wb[kUnroll];
    float sa[kUnroll], sb[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int b = b0 + u;
      if (b < nblk) {
        wa[u] = ldg_stream_u2(wrowA + b * 32 + 8 * t);
        wb[u] = ldg_stream_u2(wrowB + b * 32 + 8 * t);
        sa[u] = __ldg(arowA + b);
        sb[u] = __ldg(arowB + b);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int b = b0 + u;
      if (b >= nblk) break;
      uint32_t xf[NT8][8];
#pragma unroll
      for (int j = 0; j < NT8; ++j) {
        if (xok[j]) {
          load_x16<AT>(A, xrow[j] + (size_t)b * kBlock + 16 * t, xf[j]);
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) xf[j][q] = 0u;
        }
      }
      float tmp[NT8][4];
#pragma unroll
      for (int j = 0; j < NT8; ++j)
#pragma unroll
        for (int q = 0; q < 4; ++q) tmp[j][q] = 0.0f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        // bytes 2i and 2i+1 of this lane's 8 bytes of each row
        const uint32_t wA = (i < 2) ? wa[u].x : wa[u].y;
        const uint32_t wB = (i < 2) ? wb[u].x : wb[u].y;
        const uint32_t lo = (i & 1) * 2;
        uint32_t a[4];
        a[0] = lut[__byte_perm(wA, 0, 0x4440u | lo) * 32 + lane];
        a[1] = lut[__byte_perm(wB, 0, 0x4440u | lo) * 32 + lane];
        a[2] = lut[__byte_perm(wA, 0, 0x4440u | (lo + 1)) * 32 + lane];
        a[3] = lut[__byte_perm(wB, 0, 0x4440u | (lo + 1)) * 32 + lane];
#pragma unroll
        for (int j = 0; j < NT8; ++j) mma_f16_16816(tmp[j], a, xf[j][2 * i], xf[j][2 * i + 1]);
      }
#pragma unroll
      for (int j = 0; j < NT8; ++j) {
        acc[j][0] = fmaf(sa[u], tmp[j][0], acc[j][0]);
        acc[j][1] = fmaf(sa[u], tmp[j][1], acc[j][1]);
        acc[j][2] = fmaf(sb[u], tmp[j][2], acc[j][2]);
        acc[j][3] = fmaf(sb[u], tmp[j][3], acc[j][3]);
      }
    }
  }

  // Epilogue: D[m][n] -> out[token n][row m].  acc[j][q]: row g (q < 2) or
  // g+8 (q >= 2), token 8j + 2t + (q & 1).
#pragma unroll
  for (int j = 0; j < NT8; ++j) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int tok = 8 * j + 2 * t + q;
      if (tok >= cnt) continue;
      const size_t p = (size_t)(p0 + tok);
      if (EPI == MOE_EPI_SWIGLU) {
        store_checked(out, p * (size_t)(N / 2) + outColA, swiglu_f32(acc[j][q], acc[j][q + 2]),
                  dev_err);
      } else {
        store_checked(out, p * (size_t)N + outColA, acc[j][q], dev_err);
        store_checked(out, p * (size_t)N + outColB, acc[j][q + 2], dev_err);
      }
    }
  }
}

template <typename AT, int EPI, typename OutT>
__global__ void __launch_bounds__(32 * kWarps) gemv_nf4_kernel(
    const AT* __restrict__ A, int A_rows, const int32_t* __restrict__ gather, int k,
    const uint8_t* __restrict__ packed, const float* __restrict__ absmax,
    const int32_t* __restrict__ offsets, int E, int N, int K, int M_total,
    OutT* __restrict__ out, int32_t* dev_err) {
  __shared__ uint32_t lut[256 * 32];
  pdl_wait();
  pdl_trigger();
  const int e = blockIdx.y;
  const int start = offsets[e], end = offsets[e + 1];
  if (threadIdx.x == 0 && blockIdx.x == 0 && e == 0 &&
      (offsets[0] != 0 || offsets[E] != M_total))
    set_dev_err(dev_err, MOE_DEVERR_BAD_OFFSETS);
  if (start < 0 || end < start || end > M_total || offsets[0] != 0 || offsets[E] != M_total) {
    if (threadIdx.x == 0) set_dev_err(dev_err, MOE_DEVERR_BAD_OFFSETS);
    return;
  }
  const int cnt = end - start;
  if (cnt == 0) return;

  // byte b -> {fp16 L[b >> 4] (low half), fp16 L[b & 15] (high half)},
  // replicated so lane l reads bank l.
  for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
    const int b = i >> 5;
    const __half2 h = __halves2half2(__float2half_rn(c_levels_gemv[b >> 4]),
                                     __float2half_rn(c_levels_gemv[b & 15]));
    lut[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2;
  // Weight rows of this lane (M rows g and g+8 of the warp's 16).
  int rowA, rowB, outColA, outColB;
  if (EPI == MOE_EPI_SWIGLU) {
    const int I = N / 2;
    const int j0 = blockIdx.x * (kRowsPerCta / 2) + warp * 8 + g;
    rowA = j0;       // gate row
    rowB = I + j0;   // matching up row
    outColA = j0;
    outColB = j0;
  } else {
    rowA = blockIdx.x * kRowsPerCta + warp * 16 + g;
    rowB = rowA + 8;
    outColA = rowA;
    outColB = rowB;
  }
  const size_t rowBytes = (size_t)K / 2, rowBlocks = (size_t)K / kBlock;
  const uint8_t* wrowA = packed + ((size_t)e * N + rowA) * rowBytes;
  const uint8_t* wrowB = packed + ((size_t)e * N + rowB) * rowBytes;
  const float* arowA = absmax + ((size_t)e * N + rowA) * rowBlocks;
  const float* arowB = absmax + ((size_t)e * N + rowB) * rowBlocks;

  for (int c0 = 0; c0 < cnt; c0 += 16) {
    const int rem = cnt - c0;
    if (rem > 8)
      gemv_chunk<AT, EPI, OutT, 2>(A, A_rows, gather, k, wrowA, wrowB, arowA, arowB, lut, K, N,
                                   M_total, start + c0, min(rem, 16), outColA, outColB, out,
                                   dev_err);
    else
      gemv_chunk<AT, EPI, OutT, 1>(A, A_rows, gather, k, wrowA, wrowB, arowA, arowB, lut, K, N,
                                   M_total, start + c0, rem, outColA, outColB, out, dev_err);
  }
}

template <typename AT, int EPI>
cudaError_t launch_out(const void* A, int A_rows, const int32_t* gather, int k, const uint8_t* packed,
                       const float* absmax, const int32_t* offsets, int E, int N, int K,
                       int M_total, void* out, moe_dtype_t out_dt, int32_t* dev_err,
                       cudaStream_t s) {
  const dim3 grid(N / kRowsPerCta, E);
  const AT* a = reinterpret_cast<const AT*>(A);
  if (out_dt == MOE_DT_F32)
    return launch_pdl(gemv_nf4_kernel<AT, EPI, float>, grid, dim3(32 * kWarps), 0, s, a, A_rows,
                      gather, k, packed, absmax, offsets, E, N, K, M_total, (float*)out, dev_err);
  if (out_dt == MOE_DT_F16)
    return launch_pdl(gemv_nf4_kernel<AT, EPI, __half>, grid, dim3(32 * kWarps), 0, s, a, A_rows,
                      gather, k, packed, absmax, offsets, E, N, K, M_total, (__half*)out, dev_err);
  return launch_pdl(gemv_nf4_kernel<AT, EPI, __nv_bfloat16>, grid, dim3(32 * kWarps), 0, s, a,
                    A_rows, gather, k, packed, absmax, offsets, E, N, K, M_total,
                    (__nv_bfloat16*)out, dev_err);
}

}  // namespace
}  // namespace moe

namespace moe_launch {

cudaError_t grouped_gemm_gemv(const void* A, moe_dtype_t a_dt, int A_rows, const int32_t* gather,
                              int k,
                              const uint8_t* packed, const float* absmax,
                              const int32_t* offsets, int E, int N, int K, int M_total,
                              moe_epilogue_t epi, void* out, moe_dtype_t out_dt,
                              int32_t* dev_err, cudaStream_t s, bool chain) {
  if (M_total == 0) return cudaSuccess;
  if (!gather && a_dt == MOE_DT_F16 && grouped_gemm_decode_supported(N, K))
    return grouped_gemm_decode(A, A_rows, packed, absmax, offsets, E, N, K, M_total, epi, out,
                               out_dt, dev_err, s, chain);
  using namespace moe;
  if (a_dt == MOE_DT_BF16) {
    return epi == MOE_EPI_SWIGLU
               ? launch_out<__nv_bfloat16, MOE_EPI_SWIGLU>(A, A_rows, gather, k, packed, absmax, offsets,
                                                           E, N, K, M_total, out, out_dt,
                                                           dev_err, s)
               : launch_out<__nv_bfloat16, MOE_EPI_NONE>(A, A_rows, gather, k, packed, absmax, offsets,
                                                         E, N, K, M_total, out, out_dt,
                                                         dev_err, s);
  }
  return epi == MOE_EPI_SWIGLU
             ? launch_out<__half, MOE_EPI_SWIGLU>(A, A_rows, gather, k, packed, absmax, offsets, E, N, K,
                                                  M_total, out, out_dt, dev_err, s)
             : launch_out<__half, MOE_EPI_NONE>(A, A_rows, gather, k, packed, absmax, offsets, E, N, K,
                                                M_total, out, out_dt, dev_err, s);
}

}  // namespace moe_launch
