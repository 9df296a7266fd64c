// Grouped NF4 GEMM, decode path with TMA-staged weights (few rows per
// expert; HBM-bound).
//
// "grouped-nf4-gemm & experts-4bit" (jordananderson-pages.pages.dev), first
// bullet: one launch for all active experts, the 16-entry codebook decoded in
// registers, no dequantized weight copy.  At decode sizes the whole cost is
// streaming the NF4 bytes of every expert that received a token, so the
// design goal is to keep enough bytes in flight to saturate HBM:
//
// * Persistent CTAs (one per SM) walk a list of work items built on the
//   device from expert_offsets: (expert, 128 weight rows, up to 16 routed
//   rows; an expert with more routed rows yields one item per 16).
// * One producer thread streams each item through a 6-stage ring with TMA
//   tile loads, 256 k per stage: the packed rows (128 x 128 bytes), their
//   absmax (128 x 4 fp32) and the routed activation rows (fp16, 8-row boxes
//   of 64 k); 128-byte swizzle keeps the consumers' shared reads
//   conflict-free.  Up to ~150 KB in flight per SM, independent of registers.
// * Eight consumer warps each own 16 weight rows: per 64-k block a lane reads
//   8 packed bytes of two rows, maps each byte to an fp16 pair {L[hi], L[lo]}
//   with one lookup in a per-lane replicated table, and issues
//   mma.sync.m16n8k16 with the routed rows as the N side (swap-AB); the
//   block's fp32 absmax scales the block's fp32 partial sums.
// * The SwiGLU epilogue pairs gate row j and up row I + j in the same lane.
// Every wait is bounded; on expiry MOE_DEVERR_TIMEOUT is set and all roles
// leave their loops.
#include "common.cuh"

namespace moe {
namespace dec {

constexpr int ROWS = 128;       // weight rows per item
constexpr int TOK = 16;         // routed rows per item (max)
constexpr int SK = 256;         // k per stage
constexpr int SB = SK / 2;      // packed bytes per row per stage
constexpr int STAGES = 6;
constexpr int CWARPS = 8;
constexpr int THREADS = 32 * (CWARPS + 1);
constexpr uint32_t kSpinLimit = 1u << 24;
constexpr uint32_t kWBytes = ROWS * SB + ROWS * 4 * 4;   // packed + absmax per stage
constexpr int XBOX = 8 * 64 * 2;                         // one 8-row x 64-k fp16 box
constexpr int XKBOX = (TOK / 8) * XBOX;                  // 16 rows x 64 k

struct __align__(8) Smem {
  uint8_t w[STAGES][ROWS * SB];  // 1024-aligned (struct placed at 1024)
  uint8_t x[STAGES][4 * XKBOX];  // [64-k block][16 rows][128 B], swizzled
  float a[STAGES][ROWS * 4];
  uint32_t lut[256 * 32];
  uint64_t full[STAGES], empty[STAGES];
  int abort_flag;
  int nitems;
  int item_prefix[1025];
};

__constant__ float c_levels_dec[16] = {MOE_NF4_LEVEL_LIST};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, Smem& sm,
                                          int32_t* dev_err) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*reinterpret_cast<volatile int*>(&sm.abort_flag)) return false;
  }
  *reinterpret_cast<volatile int*>(&sm.abort_flag) = 1;
  set_dev_err(dev_err, MOE_DEVERR_TIMEOUT);
  return false;
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
      "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// This lane's 16 activations of routed row `r` (0..15) in 64-k block `b` of
// a stage, as 8 fp16 pairs: bytes [32t, 32t + 32) of the row's swizzled
// 128-byte line.
__device__ __forceinline__ void lds_x16(const uint8_t* xs, int b, int r, int t,
                                        uint32_t (&xf)[8]) {
  const uint8_t* line = xs + b * XKBOX + r * 128;
  const uint4 u = *reinterpret_cast<const uint4*>(line + (((2 * t) ^ (r & 7)) << 4));
  const uint4 v = *reinterpret_cast<const uint4*>(line + (((2 * t + 1) ^ (r & 7)) << 4));
  xf[0] = u.x; xf[1] = u.y; xf[2] = u.z; xf[3] = u.w;
  xf[4] = v.x; xf[5] = v.y; xf[6] = v.z; xf[7] = v.w;
}

struct Item {
  int expert, rtile, start, cnt;  // routed rows [start, start + cnt)
};

__device__ __forceinline__ Item item_info(const Smem& sm, const int32_t* offsets, int E,
                                          int rtiles, int it) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (sm.item_prefix[mid] <= it) lo = mid; else hi = mid;
  }
  const int local = it - sm.item_prefix[lo];
  const int tc = local / rtiles;
  Item r;
  r.expert = lo;
  r.rtile = local - tc * rtiles;
  const int s = offsets[lo], e = offsets[lo + 1];
  r.start = s + tc * TOK;
  r.cnt = min(TOK, e - r.start);
  return r;
}

// One item's main loop and epilogue for one consumer warp, NT8 token tiles.
template <int EPI, typename OutT, int NT8>
__device__ __forceinline__ bool consume_item(Smem& sm, const Item& it, int N, int K,
                                             OutT* __restrict__ out, int32_t* dev_err,
                                             int& stage, uint32_t& phase) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int rA = (EPI == MOE_EPI_SWIGLU) ? 8 * warp + g : 16 * warp + g;
  const int rB = (EPI == MOE_EPI_SWIGLU) ? ROWS / 2 + 8 * warp + g : 16 * warp + g + 8;

  float acc[NT8][4];
#pragma unroll
  for (int j = 0; j < NT8; ++j)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[j][q] = 0.0f;

  const uint32_t* lut = sm.lut + lane;
  const int KS = K / SK;
  for (int s = 0; s < KS; ++s) {
    if (!mbar_wait(&sm.full[stage], phase, sm, dev_err)) return false;
    const uint8_t* wst = sm.w[stage];
    const uint8_t* xst = sm.x[stage];
    const float4 sa = *reinterpret_cast<const float4*>(&sm.a[stage][rA * 4]);
    const float4 sb = *reinterpret_cast<const float4*>(&sm.a[stage][rB * 4]);
    const float sav[4] = {sa.x, sa.y, sa.z, sa.w};
    const float sbv[4] = {sb.x, sb.y, sb.z, sb.w};
    // Two 64-k blocks at a time, so two independent MMA chains interleave.
#pragma unroll
    for (int bp = 0; bp < 2; ++bp) {
      uint32_t xf[2][NT8][8];
      uint2 wa[2], wb[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int b = 2 * bp + h;
#pragma unroll
        for (int j = 0; j < NT8; ++j) lds_x16(xst, b, 8 * j + g, t, xf[h][j]);
        // byte offset of this lane's 8 bytes in the row, 128-byte swizzled
        const int off = b * 32 + 8 * t;
        wa[h] = *reinterpret_cast<const uint2*>(
            wst + rA * SB + ((((off >> 4) ^ (rA & 7)) << 4) | (off & 15)));
        wb[h] = *reinterpret_cast<const uint2*>(
            wst + rB * SB + ((((off >> 4) ^ (rB & 7)) << 4) | (off & 15)));
      }
      float tmp[2][NT8][4];
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int j = 0; j < NT8; ++j)
#pragma unroll
          for (int q = 0; q < 4; ++q) tmp[h][j][q] = 0.0f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t lo = (i & 1) * 2;  // byte of the word feeding slots 2t, 2t+1
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t vA = (i < 2) ? wa[h].x : wa[h].y;
          const uint32_t vB = (i < 2) ? wb[h].x : wb[h].y;
          // byte -> table entry (byte * 32 + lane): one byte_perm and one shift-add
          uint32_t af[4];
          af[0] = lut[__byte_perm(vA, 0, 0x4440u | lo) << 5];
          af[1] = lut[__byte_perm(vB, 0, 0x4440u | lo) << 5];
          af[2] = lut[__byte_perm(vA, 0, 0x4440u | (lo + 1)) << 5];
          af[3] = lut[__byte_perm(vB, 0, 0x4440u | (lo + 1)) << 5];
#pragma unroll
          for (int j = 0; j < NT8; ++j)
            mma_16816(tmp[h][j], af, xf[h][j][2 * i], xf[h][j][2 * i + 1]);
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float s_a = sav[2 * bp + h], s_b = sbv[2 * bp + h];
#pragma unroll
        for (int j = 0; j < NT8; ++j) {
          acc[j][0] = fmaf(s_a, tmp[h][j][0], acc[j][0]);
          acc[j][1] = fmaf(s_a, tmp[h][j][1], acc[j][1]);
          acc[j][2] = fmaf(s_b, tmp[h][j][2], acc[j][2]);
          acc[j][3] = fmaf(s_b, tmp[h][j][3], acc[j][3]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[stage]);
    if (++stage == STAGES) { stage = 0; phase ^= 1; }
  }

  // acc[j][q]: row rA (q < 2) or rB (q >= 2), routed row 8j + 2t + (q & 1)
#pragma unroll
  for (int j = 0; j < NT8; ++j) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int tok = 8 * j + 2 * t + q;
      if (tok >= it.cnt) continue;
      const size_t p = (size_t)(it.start + tok);
      if (EPI == MOE_EPI_SWIGLU) {
        const int I = N / 2;
        const int col = it.rtile * (ROWS / 2) + 8 * warp + g;
        out[p * I + col] = from_f32<OutT>(swiglu_f32(acc[j][q], acc[j][q + 2]));
      } else {
        const int col = it.rtile * ROWS + 16 * warp + g;
        out[p * N + col] = from_f32<OutT>(acc[j][q]);
        out[p * N + col + 8] = from_f32<OutT>(acc[j][q + 2]);
      }
    }
  }
  return true;
}

template <int EPI, typename OutT>
__global__ void __launch_bounds__(THREADS, 1) nf4_decode_kernel(
    const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap amap,
    const __grid_constant__ CUtensorMap xmap, const int32_t* __restrict__ offsets, int E, int N,
    int K, int M_total, OutT* __restrict__ out, int32_t* dev_err) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rtiles = N / ROWS;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], CWARPS);
    }
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = threadIdx.x; i < 256 * 32; i += THREADS) {
    const int b = i >> 5;
    const __half2 h = __halves2half2(__float2half_rn(c_levels_dec[b >> 4]),
                                     __float2half_rn(c_levels_dec[b & 15]));
    sm.lut[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  if (warp == CWARPS) {
    // item_prefix[e] = sum over e' < e of ceil(count / TOK) * rtiles
    bool bad = offsets[0] != 0 || offsets[E] != M_total;
    int run = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int c = 0;
      if (e < E) {
        c = offsets[e + 1] - offsets[e];
        if (c < 0) { bad = true; c = 0; }
      }
      const int items = ((c + TOK - 1) / TOK) * rtiles;
      int incl = items;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (e < E) sm.item_prefix[e] = run + incl - items;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      sm.item_prefix[E] = run;
      sm.nitems = bad ? 0 : run;
      if (bad) set_dev_err(dev_err, MOE_DEVERR_BAD_OFFSETS);
    }
  }
  __syncthreads();
  const int total = sm.nitems;
  const int KS = K / SK;

  if (warp == CWARPS) {
    // ---------------- producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = blockIdx.x; i < total && ok; i += gridDim.x) {
        const Item it = item_info(sm, offsets, E, rtiles, i);
        int y0, y1;
        if (EPI == MOE_EPI_SWIGLU) {
          y0 = it.expert * N + it.rtile * (ROWS / 2);
          y1 = y0 + N / 2;
        } else {
          y0 = it.expert * N + it.rtile * ROWS;
          y1 = y0 + ROWS / 2;
        }
        const int nr8 = (it.cnt + 7) / 8;
        for (int s = 0; s < KS; ++s) {
          if (!(ok = mbar_wait(&sm.empty[stage], phase ^ 1, sm, dev_err))) break;
          mbar_arrive_expect_tx(&sm.full[stage], kWBytes + nr8 * 4 * XBOX);
          tma_load_2d(sm.w[stage], &wmap, &sm.full[stage], s * SB, y0);
          tma_load_2d(sm.w[stage] + (ROWS / 2) * SB, &wmap, &sm.full[stage], s * SB, y1);
          tma_load_2d(sm.a[stage], &amap, &sm.full[stage], s * 4, y0);
          tma_load_2d(sm.a[stage] + (ROWS / 2) * 4, &amap, &sm.full[stage], s * 4, y1);
          for (int b = 0; b < 4; ++b)
            for (int r = 0; r < nr8; ++r)
              tma_load_2d(sm.x[stage] + b * XKBOX + r * XBOX, &xmap, &sm.full[stage],
                          s * SK + b * kBlock, it.start + 8 * r);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else {
    // ---------------- consumers
    int stage = 0;
    uint32_t phase = 0;
    for (int i = blockIdx.x; i < total; i += gridDim.x) {
      const Item it = item_info(sm, offsets, E, rtiles, i);
      bool ok;
      if (it.cnt > 8)
        ok = consume_item<EPI, OutT, 2>(sm, it, N, K, out, dev_err, stage, phase);
      else
        ok = consume_item<EPI, OutT, 1>(sm, it, N, K, out, dev_err, stage, phase);
      if (!ok) break;
    }
  }
  __syncwarp();  // the producer lane rejoins its warp before the CTA barrier
  __syncthreads();
}

int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <int EPI, typename OutT>
cudaError_t launch(const void* A, int A_rows, const uint8_t* packed, const float* absmax,
                   const int32_t* offsets, int E, int N, int K, int M_total, void* out,
                   int32_t* dev_err, cudaStream_t s) {
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap wmap, amap, xmap;
  const cuuint32_t estr[2] = {1, 1};
  {
    const cuuint64_t dims[2] = {(cuuint64_t)K / 2, (cuuint64_t)E * N};
    const cuuint64_t strides[1] = {(cuuint64_t)K / 2};
    const cuuint32_t box[2] = {SB, ROWS / 2};
    if (enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(packed), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)K / kBlock, (cuuint64_t)E * N};
    const cuuint64_t strides[1] = {(cuuint64_t)K / kBlock * 4};
    const cuuint32_t box[2] = {SK / kBlock, ROWS / 2};
    if (enc(&amap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(absmax), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)A_rows};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {kBlock, 8};
    if (enc(&xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(A), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const size_t smem = sizeof(Smem) + 1024;
  auto kern = nf4_decode_kernel<EPI, OutT>;
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int64_t max_items = ((int64_t)M_total / TOK + E) * (N / ROWS);
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(sm_count(), max_items));
  kern<<<grid, THREADS, smem, s>>>(wmap, amap, xmap, offsets, E, N, K, M_total,
                                   reinterpret_cast<OutT*>(out), dev_err);
  return cudaGetLastError();
}

template <int EPI>
cudaError_t launch_out(const void* A, int A_rows, const uint8_t* packed, const float* absmax,
                       const int32_t* offsets, int E, int N, int K, int M_total, void* out,
                       moe_dtype_t out_dt, int32_t* dev_err, cudaStream_t s) {
  if (out_dt == MOE_DT_F32)
    return launch<EPI, float>(A, A_rows, packed, absmax, offsets, E, N, K, M_total, out,
                              dev_err, s);
  if (out_dt == MOE_DT_F16)
    return launch<EPI, __half>(A, A_rows, packed, absmax, offsets, E, N, K, M_total, out,
                               dev_err, s);
  return launch<EPI, __nv_bfloat16>(A, A_rows, packed, absmax, offsets, E, N, K, M_total, out,
                                    dev_err, s);
}

}  // namespace dec
}  // namespace moe

namespace moe_launch {

bool grouped_gemm_decode_supported(int N, int K) {
  // absmax rows must be a multiple of 16 bytes for the TMA map: K % 256.
  return N % moe::dec::ROWS == 0 && K % moe::dec::SK == 0;
}

// Activations must be fp16 rows in permuted order (no gather).
cudaError_t grouped_gemm_decode(const void* A, int A_rows, const uint8_t* packed,
                                const float* absmax, const int32_t* offsets, int E, int N, int K,
                                int M_total, moe_epilogue_t epi, void* out, moe_dtype_t out_dt,
                                int32_t* dev_err, cudaStream_t s) {
  using namespace moe::dec;
  return epi == MOE_EPI_SWIGLU
             ? launch_out<MOE_EPI_SWIGLU>(A, A_rows, packed, absmax, offsets, E, N, K, M_total,
                                          out, out_dt, dev_err, s)
             : launch_out<MOE_EPI_NONE>(A, A_rows, packed, absmax, offsets, E, N, K, M_total, out,
                                        out_dt, dev_err, s);
}

}  // namespace moe_launch
