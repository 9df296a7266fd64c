// Grouped MXFP4 GEMM, decode path (few rows per expert; HBM-bound).
//
// The pages' kernel also serves MXFP4, computing on a checkpoint's exact
// released bytes ("Jordan Anderson", jordananderson-pages.pages.dev, section
// "grouped-nf4-gemm & experts-4bit", third bullet), with e2m1 elements and e8m0
// scales ("MoE Training on Consumer GPUs", cerinamroth.com/ml, section "Task
// guides").  Format (OCP Microscaling v1.0): 4-bit E2M1 codes, two per byte
// with element 2j in the LOW nibble, and per 32 consecutive elements along K
// one E8M0 scale byte b, w = 2^(b - 127) * e2m1(code).
//
// The kernel is the NF4 / INT4 decode GEMV's pipeline (persistent CTAs over
// (expert, 128 weight rows, <= 16 routed rows) items, one TMA producer, eight
// consumer warps with swap-AB mma.sync.m16n8k16).  Each packed byte becomes
// the exact fp16 pair {e2m1(low nibble), e2m1(high nibble)} through one
// byte_perm and one per-lane shared-table load.  A lane's sixteen codes of a
// row in a 64-k block all lie in one 32-element scale block, so the lane
// multiplies its fp16 pairs by that block's power of two (HMUL2), which is
// exact while 2^(b - 127) lies in [2^-23, 2^13]; scale bytes outside that
// range (other than 0, an all-zero block) set MOE_DEVERR_RANGE.  Scale bytes
// come from global memory, eight per row per 256-k stage, one stage ahead.
// Every wait is bounded; on expiry MOE_DEVERR_TIMEOUT is set and all roles
// leave their loops.
#include "common.cuh"

namespace moe {
namespace mx4 {

constexpr int ROWS = 128;       // weight rows per item
constexpr int TOK = 16;         // routed rows per item (max)
constexpr int SK = 256;         // k per stage
constexpr int SB = SK / 2;      // packed bytes per row per stage
constexpr int SBLK = 32;        // k per scale byte
constexpr int STAGES = 5;
constexpr int CWARPS = 8;
constexpr int THREADS = 32 * (CWARPS + 1);
constexpr uint32_t kSpinLimit = 1u << 24;
constexpr int XBOX = 8 * 64 * 2;                 // one 8-row x 64-k fp16 box
constexpr int XKBOX = (TOK / 8) * XBOX;          // 16 rows x 64 k
constexpr uint32_t kWBytes = ROWS * SB;          // packed rows per stage
constexpr uint32_t kXBytes = 4 * XKBOX;          // activations per stage (max)
constexpr uint32_t kStageBytes = kWBytes + kXBytes;  // 24 KB, 1 KB multiple

// Absolute shared-memory layout.  The dynamic window must start at or below
// 1 KB (checked at run time).  Stages need 1 KB alignment (128-byte swizzle).
constexpr uint32_t kStage0 = 1024;                        // stages 0-1
constexpr uint32_t kMisc = kStage0 + 2 * kStageBytes;     // barriers, item list
constexpr uint32_t kLut = 65536;                          // table: 256 x 256 B
constexpr uint32_t kStage2 = 2 * 65536;                   // stages 2-4

__device__ __forceinline__ uint32_t stage_addr(int s) {
  return s < 2 ? kStage0 + s * kStageBytes : kStage2 + (s - 2) * kStageBytes;
}

struct Misc {
  uint64_t full[STAGES], empty[STAGES];
  int abort_flag;
  int nitems;
  int item_prefix[1025];
};
static_assert(kMisc + sizeof(Misc) <= kLut, "shared layout overlap");
constexpr uint32_t kEnd = kStage2 + (STAGES - 2) * kStageBytes;
static_assert(kEnd <= 227 * 1024, "shared layout too large");

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, Misc& ms,
                                          int32_t* dev_err) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*reinterpret_cast<volatile int*>(&ms.abort_flag)) return false;
  }
  *reinterpret_cast<volatile int*>(&ms.abort_flag) = 1;
  set_dev_err(dev_err, MOE_DEVERR_TIMEOUT);
  return false;
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a));
  return v;
}

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
      "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
struct Item {
  int expert, rtile, start, cnt;  // routed rows [start, start + cnt)
};

__device__ __forceinline__ Item item_info(const Misc& ms, const int32_t* offsets, int E,
                                          int rtiles, int it) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (ms.item_prefix[mid] <= it) lo = mid; else hi = mid;
  }
  const int local = it - ms.item_prefix[lo];
  const int tc = local / rtiles;
  Item r;
  r.expert = lo;
  r.rtile = local - tc * rtiles;
  const int s = offsets[lo], e = offsets[lo + 1];
  r.start = s + tc * TOK;
  r.cnt = min(TOK, e - r.start);
  return r;
}

__device__ __forceinline__ uint32_t mul_h2(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// One item's main loop and epilogue for one consumer warp, NT8 token tiles.
template <int EPI, typename OutT, int NT8>
__device__ __forceinline__ bool consume_item(Misc& ms, const Item& it, int N, int K,
                                             const uint8_t* __restrict__ scales,
                                             OutT* __restrict__ out, int32_t* dev_err,
                                             int& stage, uint32_t& phase) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int sg = ((g & 3) << 1) | (g >> 2);  // sigma(g)
  const int rA = (EPI == MOE_EPI_SWIGLU) ? 8 * warp + sg : 16 * warp + sg;
  const int rB = (EPI == MOE_EPI_SWIGLU) ? ROWS / 2 + 8 * warp + sg : 16 * warp + sg + 8;
  // global weight rows of rA, rB (SwiGLU tiles: gate rows, then up rows N/2 on)
  const int gA = (EPI == MOE_EPI_SWIGLU) ? it.rtile * (ROWS / 2) + rA : it.rtile * ROWS + rA;
  const int gB = (EPI == MOE_EPI_SWIGLU) ? N / 2 + it.rtile * (ROWS / 2) + (rB - ROWS / 2)
                                         : it.rtile * ROWS + rB;
  const int KB = K / SBLK;
  // eight scale bytes per row per 256-k stage
  const uint2* mpA = reinterpret_cast<const uint2*>(scales + ((size_t)it.expert * N + gA) * KB);
  const uint2* mpB = reinterpret_cast<const uint2*>(scales + ((size_t)it.expert * N + gB) * KB);
  bool bad_scale = false;
  // byte_perm source: 0x10000 | lane << 2 -> entry address of a byte
  const uint32_t lb = 0x10000u | ((uint32_t)lane << 2);
  // this lane's 8 packed bytes of block b in a 128-byte swizzled row whose
  // row index is congruent to sg (mod 8): chunk (2b + t/2) ^ sg, half t & 1
  uint32_t woff[4];
#pragma unroll
  for (int b = 0; b < 4; ++b)
    woff[b] = ((((2 * b + (t >> 1)) ^ sg) << 4) | ((t & 1) << 3));
  // activation rows 8j + g: chunks 2t and 2t+1 of the 128-byte line, swizzled
  const uint32_t xo0 = (uint32_t)(((2 * t) ^ g) << 4), xo1 = (uint32_t)(((2 * t + 1) ^ g) << 4);

  float acc[NT8][4];
#pragma unroll
  for (int j = 0; j < NT8; ++j)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[j][q] = 0.0f;

  const int KS = K / SK;
  // the stage's eight scale bytes of rows rA and rB, one stage ahead
  uint2 mA = __ldg(mpA), mB = __ldg(mpB);
  for (int s = 0; s < KS; ++s) {
    const uint2 nA = (s + 1 < KS) ? __ldg(mpA + s + 1) : make_uint2(0, 0);
    const uint2 nB = (s + 1 < KS) ? __ldg(mpB + s + 1) : make_uint2(0, 0);
    const uint32_t base = stage_addr(stage);
    if (!mbar_wait(smem_u32(&ms.full[stage]), phase, ms, dev_err)) return false;
    const uint32_t wst = base, xst = base + kWBytes;
    const uint32_t mAv[2] = {mA.x, mA.y}, mBv[2] = {mB.x, mB.y};
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      // this lane's codes of block b lie in scale block 2b + t/2 of the stage
      const int sbi = 2 * b + (t >> 1);
      const uint32_t bA = (mAv[sbi >> 2] >> (8 * (sbi & 3))) & 0xFFu;
      const uint32_t bB = (mBv[sbi >> 2] >> (8 * (sbi & 3))) & 0xFFu;
      const uint32_t zA = mx_scale_h2(bA, bad_scale);
      const uint32_t zB = mx_scale_h2(bB, bad_scale);
      uint32_t xf[NT8][8];
#pragma unroll
      for (int j = 0; j < NT8; ++j) {
        const uint32_t line = xst + b * XKBOX + (8 * j + g) * 128;
        const uint4 u = lds128(line + xo0), v = lds128(line + xo1);
        xf[j][0] = u.x; xf[j][1] = u.y; xf[j][2] = u.z; xf[j][3] = u.w;
        xf[j][4] = v.x; xf[j][5] = v.y; xf[j][6] = v.z; xf[j][7] = v.w;
      }
      const uint2 wa = lds64(wst + rA * SB + woff[b]);
      const uint2 wb = lds64(wst + rB * SB + woff[b]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t lo = (i & 1) * 2;  // byte of the word feeding slots 2t, 2t+1
        const uint32_t s0 = 0x7604u | (lo << 4), s1 = 0x7604u | ((lo + 1) << 4);
        const uint32_t vA = (i < 2) ? wa.x : wa.y, vB = (i < 2) ? wb.x : wb.y;
        uint32_t af[4];
        af[0] = mul_h2(lds32(__byte_perm(vA, lb, s0)), zA);
        af[1] = mul_h2(lds32(__byte_perm(vB, lb, s0)), zB);
        af[2] = mul_h2(lds32(__byte_perm(vA, lb, s1)), zA);
        af[3] = mul_h2(lds32(__byte_perm(vB, lb, s1)), zB);
#pragma unroll
        for (int j = 0; j < NT8; ++j) mma_16816(acc[j], af, xf[j][2 * i], xf[j][2 * i + 1]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&ms.empty[stage]));
    if (++stage == STAGES) { stage = 0; phase ^= 1; }
    mA = nA;
    mB = nB;
  }

  if (bad_scale) set_dev_err(dev_err, MOE_DEVERR_RANGE);
  // acc[j][q]: row rA (q < 2) or rB (q >= 2), routed row 8j + 2t + (q & 1)
#pragma unroll
  for (int j = 0; j < NT8; ++j) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int tok = 8 * j + 2 * t + q;
      if (tok >= it.cnt) continue;
      const size_t p = (size_t)(it.start + tok);
      if (EPI == MOE_EPI_SWIGLU) {
        store_checked(out, p * (N / 2) + gA, swiglu_f32(acc[j][q], acc[j][q + 2]), dev_err);
      } else {
        store_checked(out, p * N + gA, acc[j][q], dev_err);
        store_checked(out, p * N + gB, acc[j][q + 2], dev_err);
      }
    }
  }
  return true;
}

template <int EPI, typename OutT>
__global__ void __launch_bounds__(THREADS, 1) mxfp4_decode_kernel(
    const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap,
    const uint8_t* __restrict__ scales, const int32_t* __restrict__ offsets, int E, int N, int K,
    int M_total, OutT* __restrict__ out, int32_t* dev_err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  if (base > kStage0) {  // layout assumption broken: do nothing, say so
    if (threadIdx.x == 0) set_dev_err(dev_err, MOE_DEVERR_LAYOUT);
    return;
  }
  Misc& ms = *reinterpret_cast<Misc*>(smem_raw + (kMisc - base));
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem_raw + (kLut - base));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rtiles = N / ROWS;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&ms.full[s]), 1);
      mbar_init(smem_u32(&ms.empty[s]), CWARPS);
    }
    ms.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // byte b -> {fp16 e2m1(b & 15) (low half), fp16 e2m1(b >> 4) (high half)},
  // one 256-byte row per byte value, lane l's copy at 4 l.  fp16 bits of the
  // E2M1 magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; bit 3 of a code is its sign.
  for (int i = threadIdx.x; i < 256 * 32; i += THREADS) {
    const uint32_t b = (uint32_t)(i >> 5), l = (uint32_t)(i & 31);
    lut[b * 64 + l] = e2m1_h(b & 15u) | (e2m1_h(b >> 4) << 16);
  }
  if (warp == CWARPS) {
    // item_prefix[e] = sum over e' < e of ceil(count / TOK) * rtiles
    bool bad = offsets[0] != 0 || offsets[E] != M_total;
    int run = 0;
    for (int b0 = 0; b0 < E; b0 += 32) {
      const int e = b0 + lane;
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
      if (e < E) ms.item_prefix[e] = run + incl - items;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      ms.item_prefix[E] = run;
      ms.nitems = bad ? 0 : run;
      if (bad) set_dev_err(dev_err, MOE_DEVERR_BAD_OFFSETS);
    }
  }
  __syncthreads();
  const int total = ms.nitems;
  const int KS = K / SK;

  if (warp == CWARPS) {
    // ---------------- producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = blockIdx.x; i < total && ok; i += gridDim.x) {
        const Item it = item_info(ms, offsets, E, rtiles, i);
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
          const uint32_t full = smem_u32(&ms.full[stage]);
          if (!(ok = mbar_wait(smem_u32(&ms.empty[stage]), phase ^ 1, ms, dev_err))) break;
          const uint32_t sb = stage_addr(stage);
          mbar_arrive_expect_tx(full, kWBytes + nr8 * 4 * XBOX);
          tma_load_2d(sb, &wmap, full, s * SB, y0);
          tma_load_2d(sb + (ROWS / 2) * SB, &wmap, full, s * SB, y1);
          for (int b = 0; b < 4; ++b)
            for (int r = 0; r < nr8; ++r)
              tma_load_2d(sb + kWBytes + b * XKBOX + r * XBOX, &xmap, full, s * SK + b * kBlock,
                          it.start + 8 * r);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else {
    // ---------------- consumers
    int stage = 0;
    uint32_t phase = 0;
    for (int i = blockIdx.x; i < total; i += gridDim.x) {
      const Item it = item_info(ms, offsets, E, rtiles, i);
      bool ok;
      if (it.cnt > 8)
        ok = consume_item<EPI, OutT, 2>(ms, it, N, K, scales, out, dev_err, stage, phase);
      else
        ok = consume_item<EPI, OutT, 1>(ms, it, N, K, scales, out, dev_err, stage, phase);
      if (!ok) break;
    }
  }
  __syncwarp();  // the producer lane rejoins its warp before the CTA barrier
  __syncthreads();
}

int sm_count() { return device_sm_count(); }

template <int EPI, typename OutT>
cudaError_t launch(const void* A, int A_rows, const uint8_t* packed, const uint8_t* scales,
                   const int32_t* offsets, int E, int N, int K, int M_total, void* out,
                   int32_t* dev_err, cudaStream_t s) {
  if (!tensor_map_encoder()) return cudaErrorNotSupported;
  const auto enc = encode_tiled_cached;
  CUtensorMap wmap, xmap;
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
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)A_rows};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {kBlock, 8};
    if (enc(&xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(A), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const size_t smem = kEnd;  // absolute layout; the window starts at or below 1 KB
  auto kern = mxfp4_decode_kernel<EPI, OutT>;
  cudaError_t err = set_max_dynamic_smem_once(reinterpret_cast<const void*>(kern), (int)smem);
  if (err != cudaSuccess) return err;
  const int64_t max_items = ((int64_t)M_total / TOK + E) * (N / ROWS);
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(sm_count(), max_items));
  kern<<<grid, THREADS, smem, s>>>(wmap, xmap, scales, offsets, E, N, K, M_total,
                                   reinterpret_cast<OutT*>(out), dev_err);
  return cudaGetLastError();
}

template <int EPI>
cudaError_t launch_out(const void* A, int A_rows, const uint8_t* packed, const uint8_t* scales,
                       const int32_t* offsets, int E, int N, int K, int M_total, void* out,
                       moe_dtype_t out_dt, int32_t* dev_err, cudaStream_t s) {
  if (out_dt == MOE_DT_F32)
    return launch<EPI, float>(A, A_rows, packed, scales, offsets, E, N, K, M_total, out, dev_err,
                              s);
  if (out_dt == MOE_DT_F16)
    return launch<EPI, __half>(A, A_rows, packed, scales, offsets, E, N, K, M_total, out, dev_err,
                               s);
  return launch<EPI, __nv_bfloat16>(A, A_rows, packed, scales, offsets, E, N, K, M_total, out,
                                    dev_err, s);
}

}  // namespace mx4
}  // namespace moe

namespace moe_launch {

bool grouped_gemm_mxfp4_supported(int N, int K) {
  return N % moe::mx4::ROWS == 0 && K % moe::mx4::SK == 0;
}

cudaError_t grouped_gemm_mxfp4(const void* A, int A_rows, const uint8_t* packed,
                               const uint8_t* scales, const int32_t* offsets, int E, int N, int K,
                               int M_total, moe_epilogue_t epi, void* out, moe_dtype_t out_dt,
                               int32_t* dev_err, cudaStream_t s) {
  using namespace moe::mx4;
  return epi == MOE_EPI_SWIGLU
             ? launch_out<MOE_EPI_SWIGLU>(A, A_rows, packed, scales, offsets, E, N, K, M_total,
                                          out, out_dt, dev_err, s)
             : launch_out<MOE_EPI_NONE>(A, A_rows, packed, scales, offsets, E, N, K, M_total, out,
                                        out_dt, dev_err, s);
}

}  // namespace moe_launch
