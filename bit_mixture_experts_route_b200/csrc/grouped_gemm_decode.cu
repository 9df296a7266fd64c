// Grouped 4-bit GEMM, decode path (few routed rows per expert; HBM-bound):
// one pipeline for the three weight formats.
//
// "grouped-nf4-gemm & experts-4bit" (jordananderson-pages.pages.dev), first
// bullet: one launch for all active experts, the codebook decoded in
// registers, no dequantized weight copy; third bullet: the same kernel runs on
// the released MXFP4 bytes and on GPTQ-style INT4 experts.  At decode sizes
// the whole cost is streaming the packed bytes of every expert that received
// a token, so the kernel is built to keep HBM busy.
//
// Formats (FMT):
//   NF4    two codes per byte (even element in the HIGH nibble), fp32 absmax
//          per 64 along K; w = L[code] * absmax.
//   MXFP4  two E2M1 codes per byte (even element in the LOW nibble), one E8M0
//          byte b per 32 along K; w = 2^(b - 127) * e2m1(code).
//   INT4   two codes per byte (even element in the high nibble), per 128 along
//          K an fp16 scale s and a 4-bit zero z (meta word s | z << 16);
//          w = (q - z) * s.
//
// * Persistent CTAs (one per SM) walk a list of work items built on the
//   device from expert_offsets: (expert, 128 weight rows, up to 16 routed
//   rows; an expert with more routed rows yields one item per 16).
// * Two consumer groups of four warps take alternate items of the CTA's list,
//   each through its own ring of stage slots (three and two of five).  One
//   producer thread serves both rings, polling whichever group's next slot is
//   free, with TMA tile loads, 256 k per stage: the packed rows (one 3-D box of
//   2 x 64 rows x 128 bytes), for NF4 their absmax (one 3-D box of 2 x 64 rows
//   x 4 fp32) and the routed activation rows (one 3-D box of the stage's four
//   64-k blocks x 8 or 16 rows), with 128-byte swizzle: three copies per
//   stage.
// * The four warps of a group each own 32 weight rows of the item (two m-tiles
//   of 16) and run mma.sync.m16n8k16 with the weights as the M side and the
//   routed rows as N (swap-AB); the four 64-k blocks of a stage run as four
//   interleaved MMA chains.
// * NF4 and INT4: a lane turns each packed byte into an fp16 pair through ONE
//   byte_perm (which assembles the shared address of the byte's entry in a
//   per-lane table: 0x10000 | byte << 8 | lane << 2) and one shared load; the
//   table sits at shared address 64 KB, one 256-byte row per byte value, so
//   the lookups never conflict.  MXFP4: the hardware E2M1 -> fp16 conversion,
//   one instruction per byte and no table.
// * Shared-memory bandwidth bounds the consumers: per weight the table entry
//   (2 bytes), the packed code, the activation fragments and the TMA writes.
//   A warp reads a stage's activation fragments once for both of its m-tiles,
//   which halves their share against 16 rows per warp.
// * Scales: NF4 scales each 64-k block's fp32 partial sum by the row's fp32
//   absmax (the only weight rounding is the levels' fp16 one); INT4 subtracts
//   the zero in fp16 (exact) and scales the block's fp32 partial sum by s;
//   MXFP4 multiplies the fp16 pairs by the block's power of two (exact while
//   2^(b - 127) lies in [2^-23, 2^13]; scale bytes outside that range, other
//   than 0, set MOE_DEVERR_RANGE).  INT4 and MXFP4 scales come from global
//   memory, one stage ahead.
// * MMA row g of a warp maps to weight row sigma(g) = 2(g mod 4) + g div 4,
//   which makes the swizzled 8-byte reads of the packed rows conflict-free;
//   the k order inside a block is permuted the same way on both operands (a
//   lane's 8 packed bytes are 16 consecutive k).
// * The SwiGLU epilogue pairs gate row j and up row I + j in the same lane.
// Every wait is bounded; on expiry MOE_DEVERR_TIMEOUT is set and all roles
// leave their loops.
#include "common.cuh"

namespace moe {
namespace dec {

constexpr int ROWS = 128;       // weight rows per item
constexpr int TOK = 16;         // routed rows per item (max)
constexpr int SK = 256;         // k per stage
constexpr int kNAlign = 128;    // N granularity of the entry points (as the tensor-core form)
constexpr int SB = SK / 2;      // packed bytes per row per stage
constexpr int MT = 2;           // m-tiles (16 weight rows each) per consumer warp
constexpr int CWARPS = ROWS / (16 * MT);  // consumer warps per group
constexpr int GROUPS = 2;       // consumer groups, each on its own items and ring
constexpr int NSLOTS = 5;       // stage slots, both groups
constexpr int kLoSlots = 2;     // slots below the table
constexpr int PWARP = GROUPS * CWARPS;           // the producer warp
constexpr int THREADS = 32 * (PWARP + 1);
constexpr uint32_t kSpinLimit = 1u << 24;
constexpr int XBOX = 8 * 64 * 2;                 // one 8-row x 64-k fp16 box
constexpr int XKBOX = (TOK / 8) * XBOX;          // 16 rows x 64 k
constexpr uint32_t kWBytes = ROWS * SB;          // packed rows per stage
constexpr uint32_t kXBytes = 4 * XKBOX;          // activations per stage (max)
constexpr uint32_t kABytes = ROWS * 16;          // NF4 absmax per stage
constexpr int MX_BLK = 32;                       // MXFP4: k per scale byte
constexpr int I4_GROUP = 128;                    // INT4: k per scale / zero

template <int FMT>
struct Layout {
  static constexpr uint32_t kA = FMT == kFmtNF4 ? kABytes : 0;
  static constexpr uint32_t kStageBytes = kWBytes + kXBytes + kA;  // 1 KB multiple
  // Absolute shared-memory layout.  The dynamic window must start at or
  // below 1 KB (checked at run time).  Stages need 1 KB alignment (128-byte
  // swizzle).
  static constexpr uint32_t kStage0 = 1024;                            // low slots
  static constexpr uint32_t kMisc = kStage0 + kLoSlots * kStageBytes;  // barriers, item list
  static constexpr uint32_t kLut = 65536;                              // table: 256 x 256 B
  static constexpr uint32_t kStage2 = 2 * 65536;                       // high slots
  static constexpr uint32_t kEnd = kStage2 + (NSLOTS - kLoSlots) * kStageBytes;
  static __host__ __device__ constexpr uint32_t slot_addr(int slot) {
    return slot < kLoSlots ? kStage0 + slot * kStageBytes
                           : kStage2 + (slot - kLoSlots) * kStageBytes;
  }
};

struct Misc {
  uint64_t full[NSLOTS], empty[NSLOTS];
  int abort_flag;
  int nitems;
  int item_prefix[1025];
  int off[1025];  // expert_offsets, copied once (item lookups never touch global memory)
  int pre[GROUPS];  // stages of each ring's first round issued during the set-up
};
static_assert(Layout<kFmtNF4>::kMisc + sizeof(Misc) <= Layout<kFmtNF4>::kLut,
              "shared layout overlap");
static_assert(Layout<kFmtNF4>::kEnd <= 227 * 1024 + 1024, "shared layout too large");
static_assert(Layout<kFmtINT4>::kEnd <= 227 * 1024 + 1024, "shared layout too large");

// Ring slots of consumer group g: [ring_base(g), ring_base(g) + ring_size(g)),
// consecutive runs of ceil(NSLOTS / GROUPS) slots (the last run may be shorter).
constexpr int kPerGroup = (NSLOTS + GROUPS - 1) / GROUPS;
static_assert(NSLOTS - (GROUPS - 1) * kPerGroup >= 2, "every ring needs two slots");
__host__ __device__ constexpr int ring_base(int g) { return g * kPerGroup; }
__host__ __device__ constexpr int ring_size(int g) {
  return NSLOTS - g * kPerGroup < kPerGroup ? NSLOTS - g * kPerGroup : kPerGroup;
}

__constant__ float c_levels_dec[16] = {MOE_NF4_LEVEL_LIST};

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
// Non-blocking probe of a phase (the producer polls several rings).
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
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
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
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
__device__ __forceinline__ uint32_t hmul2_u(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t hsub2_u(uint32_t a, uint32_t b) {
  __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// The four bytes of w, each two E2M1 codes, as four fp16 pairs (the low
// nibble in the low half), by the hardware conversion.
__device__ __forceinline__ void e2m1x8_to_h2(uint32_t w, uint32_t (&d)[4]) {
  asm("{\n\t.reg .b8 c0, c1, c2, c3;\n\t"
      "mov.b32 {c0, c1, c2, c3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, c0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, c1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, c2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, c3;\n\t}"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(w));
}

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
      "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Same with a zero accumulator input (first MMA of a block).
__device__ __forceinline__ void mma_16816_z(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                            uint32_t b1) {
  const float z = 0.0f;
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
      "{%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(z));
}

struct Item {
  int expert, rtile, start, cnt;  // routed rows [start, start + cnt)
};

__device__ __forceinline__ Item item_info(const Misc& ms, int E, int rtiles, int it) {
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
  const int s = ms.off[lo], e = ms.off[lo + 1];
  r.start = s + tc * TOK;
  r.cnt = min(TOK, e - r.start);
  return r;
}

// Weight row (within the expert's N rows) of stage-local row r of rtile.
template <int EPI>
__device__ __forceinline__ int weight_row(int r, int rtile, int N) {
  if (EPI == MOE_EPI_SWIGLU)
    return r < ROWS / 2 ? rtile * (ROWS / 2) + r : N / 2 + rtile * (ROWS / 2) + (r - ROWS / 2);
  return rtile * ROWS + r;
}

// One item for one consumer warp, NT8 token tiles.  Warp w (w-th of its
// group) owns MT m-tiles of 16 weight rows; m-tile m holds the rows of
// "virtual warp" v = MT w + m (SwiGLU: gate rows 8 v .. 8 v + 7 and the
// matching up rows; plain: rows 16 v .. 16 v + 15).  It takes all four 64-k
// blocks of every stage (four independent MMA chains per token tile) and reads
// the stage's activation fragments once for its MT m-tiles.  The group's ring
// is slots [rbase, rbase + rsize).  Returns false if a wait gave up.
template <int FMT, int EPI, typename OutT, int NT8>
__device__ __forceinline__ bool consume_item(Misc& ms, const Item& it, int N, int K,
                                             const void* __restrict__ gscales,
                                             OutT* __restrict__ out, int32_t* dev_err,
                                             int warp, int rbase, int rsize, int& stage,
                                             uint32_t& phase) {
  using LY = Layout<FMT>;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int sg = ((g & 3) << 1) | (g >> 2);  // sigma(g)
  int rA[MT], rB[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    const int v = MT * warp + m;
    rA[m] = (EPI == MOE_EPI_SWIGLU) ? 8 * v + sg : 16 * v + sg;
    rB[m] = (EPI == MOE_EPI_SWIGLU) ? ROWS / 2 + 8 * v + sg : 16 * v + sg + 8;
  }
  // byte_perm source: 0x10000 | lane << 2 -> entry address of a byte
  const uint32_t lb = 0x10000u | ((uint32_t)lane << 2);
  // this lane's 8 packed bytes of block b in a 128-byte swizzled row whose
  // row index is congruent to sg (mod 8): chunk (2b + t/2) ^ sg, half t & 1
  uint32_t woff[4];
#pragma unroll
  for (int b = 0; b < 4; ++b) woff[b] = ((((2 * b + (t >> 1)) ^ sg) << 4) | ((t & 1) << 3));
  // activation rows 8j + g: chunks 2t and 2t+1 of a block's 128-byte line
  const uint32_t xo0 = (uint32_t)(((2 * t) ^ g) << 4), xo1 = (uint32_t)(((2 * t + 1) ^ g) << 4);

  // INT4 / MXFP4 scales of rows rA and rB from global memory, one stage
  // ahead: INT4 the meta words of the stage's two 128-k groups, MXFP4 the
  // stage's eight scale bytes
  size_t gA[MT], gB[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    gA[m] = (size_t)it.expert * N + weight_row<EPI>(rA[m], it.rtile, N);
    gB[m] = (size_t)it.expert * N + weight_row<EPI>(rB[m], it.rtile, N);
  }
  auto fetch = [&](int s, uint2 (&mA)[MT], uint2 (&mB)[MT]) {
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (FMT == kFmtINT4) {
        const uint2* p = reinterpret_cast<const uint2*>(static_cast<const uint32_t*>(gscales));
        mA[m] = __ldg(p + gA[m] * (K / I4_GROUP / 2) + s);
        mB[m] = __ldg(p + gB[m] * (K / I4_GROUP / 2) + s);
      } else if (FMT == kFmtMXFP4) {
        const uint2* p = reinterpret_cast<const uint2*>(static_cast<const uint8_t*>(gscales));
        mA[m] = __ldg(p + gA[m] * (K / MX_BLK / 8) + s);
        mB[m] = __ldg(p + gB[m] * (K / MX_BLK / 8) + s);
      }
    }
  };

  float acc[MT][NT8][4];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int j = 0; j < NT8; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[m][j][q] = 0.0f;

  bool bad_scale = false;
  const int KS = K / SK;
  uint2 cA[MT], cB[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) cA[m] = cB[m] = make_uint2(0, 0);
  if (FMT != kFmtNF4) fetch(0, cA, cB);
  for (int s = 0; s < KS; ++s) {
    uint2 nA[MT], nB[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) nA[m] = nB[m] = make_uint2(0, 0);
    if (FMT != kFmtNF4 && s + 1 < KS) fetch(s + 1, nA, nB);
    const int slot = rbase + stage;
    const uint32_t base = LY::slot_addr(slot);
    if (!mbar_wait(smem_u32(&ms.full[slot]), phase, ms, dev_err)) return false;
    const uint32_t wst = base, xst = base + kWBytes, ast = base + kWBytes + kXBytes;
    // the stage's activation fragments, shared by the warp's m-tiles
    uint32_t xf[4][NT8][8];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
#pragma unroll
      for (int j = 0; j < NT8; ++j) {
        const uint32_t line = xst + b * (NT8 * XBOX) + (8 * j + g) * 128;
        const uint4 u = lds128(line + xo0), v = lds128(line + xo1);
        xf[b][j][0] = u.x; xf[b][j][1] = u.y; xf[b][j][2] = u.z; xf[b][j][3] = u.w;
        xf[b][j][4] = v.x; xf[b][j][5] = v.y; xf[b][j][6] = v.z; xf[b][j][7] = v.w;
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      // per block b: the fp32 factor of its partial sums (NF4 absmax, INT4 s)
      // and the fp16-pair operand transform (INT4 {1024 + z}, MXFP4 2^(e-127))
      float fA[4] = {1.f, 1.f, 1.f, 1.f}, fB[4] = {1.f, 1.f, 1.f, 1.f};
      uint32_t zA[4] = {0, 0, 0, 0}, zB[4] = {0, 0, 0, 0};
      if (FMT == kFmtNF4) {
        const uint4 sa = lds128(ast + rA[m] * 16), sb = lds128(ast + rB[m] * 16);
        fA[0] = __uint_as_float(sa.x); fA[1] = __uint_as_float(sa.y);
        fA[2] = __uint_as_float(sa.z); fA[3] = __uint_as_float(sa.w);
        fB[0] = __uint_as_float(sb.x); fB[1] = __uint_as_float(sb.y);
        fB[2] = __uint_as_float(sb.z); fB[3] = __uint_as_float(sb.w);
      } else if (FMT == kFmtINT4) {
        const uint32_t mA[2] = {cA[m].x, cA[m].y}, mB[2] = {cB[m].x, cB[m].y};
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const uint32_t a = mA[b >> 1], c = mB[b >> 1];  // group of this 64-k block
          fA[b] = __half2float(__ushort_as_half((unsigned short)(a & 0xFFFFu)));
          fB[b] = __half2float(__ushort_as_half((unsigned short)(c & 0xFFFFu)));
          zA[b] = 0x64006400u | ((a >> 16) & 0xFu) * 0x00010001u;
          zB[b] = 0x64006400u | ((c >> 16) & 0xFu) * 0x00010001u;
        }
      } else {
        const uint32_t mA[2] = {cA[m].x, cA[m].y}, mB[2] = {cB[m].x, cB[m].y};
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          // a lane's 16 k of block b lie in scale block 2b + t/2 of the stage
          const int sbi = 2 * b + (t >> 1);
          zA[b] = mx_scale_h2((mA[sbi >> 2] >> (8 * (sbi & 3))) & 0xFFu, bad_scale);
          zB[b] = mx_scale_h2((mB[sbi >> 2] >> (8 * (sbi & 3))) & 0xFFu, bad_scale);
        }
      }
      uint2 wa[4], wb[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        wa[b] = lds64(wst + rA[m] * SB + woff[b]);
        wb[b] = lds64(wst + rB[m] * SB + woff[b]);
      }
      if (FMT == kFmtMXFP4) {
        // MXFP4: codes to fp16 pairs by the hardware conversion (no table),
        // times the block's power of two, straight into the accumulators
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          uint32_t pa[8], pb[8];  // fp16 pairs of bytes 0..7 of rows rA, rB in block b
          e2m1x8_to_h2(wa[b].x, *reinterpret_cast<uint32_t(*)[4]>(&pa[0]));
          e2m1x8_to_h2(wa[b].y, *reinterpret_cast<uint32_t(*)[4]>(&pa[4]));
          e2m1x8_to_h2(wb[b].x, *reinterpret_cast<uint32_t(*)[4]>(&pb[0]));
          e2m1x8_to_h2(wb[b].y, *reinterpret_cast<uint32_t(*)[4]>(&pb[4]));
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int lo = (i >> 1) * 4 + (i & 1) * 2;  // byte feeding slots 2t, 2t+1
            uint32_t af[4];
            af[0] = hmul2_u(pa[lo], zA[b]);
            af[1] = hmul2_u(pb[lo], zB[b]);
            af[2] = hmul2_u(pa[lo + 1], zA[b]);
            af[3] = hmul2_u(pb[lo + 1], zB[b]);
#pragma unroll
            for (int j = 0; j < NT8; ++j)
              mma_16816(acc[m][j], af, xf[b][j][2 * i], xf[b][j][2 * i + 1]);
          }
        }
      } else {
        float tmp[4][NT8][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t lo = (i & 1) * 2;  // byte of the word feeding slots 2t, 2t+1
          const uint32_t s0 = 0x7604u | (lo << 4), s1 = 0x7604u | ((lo + 1) << 4);
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const uint32_t vA = (i < 2) ? wa[b].x : wa[b].y;
            const uint32_t vB = (i < 2) ? wb[b].x : wb[b].y;
            uint32_t af[4];
            af[0] = lds32(__byte_perm(vA, lb, s0));
            af[1] = lds32(__byte_perm(vB, lb, s0));
            af[2] = lds32(__byte_perm(vA, lb, s1));
            af[3] = lds32(__byte_perm(vB, lb, s1));
            if (FMT == kFmtINT4) {
              af[0] = hsub2_u(af[0], zA[b]); af[2] = hsub2_u(af[2], zA[b]);
              af[1] = hsub2_u(af[1], zB[b]); af[3] = hsub2_u(af[3], zB[b]);
            }
#pragma unroll
            for (int j = 0; j < NT8; ++j) {
              if (i == 0)
                mma_16816_z(tmp[b][j], af, xf[b][j][0], xf[b][j][1]);
              else
                mma_16816(tmp[b][j], af, xf[b][j][2 * i], xf[b][j][2 * i + 1]);
            }
          }
        }
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
          for (int j = 0; j < NT8; ++j) {
            acc[m][j][0] = fmaf(fA[b], tmp[b][j][0], acc[m][j][0]);
            acc[m][j][1] = fmaf(fA[b], tmp[b][j][1], acc[m][j][1]);
            acc[m][j][2] = fmaf(fB[b], tmp[b][j][2], acc[m][j][2]);
            acc[m][j][3] = fmaf(fB[b], tmp[b][j][3], acc[m][j][3]);
          }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&ms.empty[slot]));
    if (++stage == rsize) { stage = 0; phase ^= 1; }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      cA[m] = nA[m];
      cB[m] = nB[m];
    }
  }
  if (bad_scale) set_dev_err(dev_err, MOE_DEVERR_RANGE);

  // acc[m][j][q]: row rA[m] (q < 2) or rB[m] (q >= 2), routed row 8j + 2t + (q & 1)
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int j = 0; j < NT8; ++j) {
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int tok = 8 * j + 2 * t + q;
        if (tok >= it.cnt) continue;
        const size_t p = (size_t)(it.start + tok);
        if (EPI == MOE_EPI_SWIGLU) {
          store_checked(out, p * (N / 2) + it.rtile * (ROWS / 2) + rA[m],
                        swiglu_f32(acc[m][j][q], acc[m][j][q + 2]), dev_err);
        } else {
          store_checked(out, p * N + it.rtile * ROWS + rA[m], acc[m][j][q], dev_err);
          store_checked(out, p * N + it.rtile * ROWS + rB[m], acc[m][j][q + 2], dev_err);
        }
      }
    }
  return true;
}

template <int FMT, int EPI, typename OutT>
__global__ void __launch_bounds__(THREADS, 1) decode_kernel(
    const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap amap,
    const __grid_constant__ CUtensorMap xmap8, const __grid_constant__ CUtensorMap xmap16,
    const void* __restrict__ gscales, const int32_t* __restrict__ offsets, int E, int N, int K,
    int M_total, OutT* __restrict__ out, int32_t* dev_err, int chain) {
  using LY = Layout<FMT>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  if (base > LY::kStage0) {  // layout assumption broken: do nothing, say so
    if (threadIdx.x == 0) set_dev_err(dev_err, MOE_DEVERR_LAYOUT);
    return;
  }
  Misc& ms = *reinterpret_cast<Misc*>(smem_raw + (LY::kMisc - base));
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem_raw + (LY::kLut - base));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rtiles = N / ROWS;
  const int KS = K / SK;
  const int step = GROUPS * gridDim.x;  // group g takes the CTA's items g, g + GROUPS, ...
  // the item's 128 weight rows as two 64-row halves (y, z .. z+1) of the 3-D
  // weight (and absmax) maps: SwiGLU items take the gate rows and the
  // matching up rows (z = 2e + half), plain items 128 consecutive rows
  auto rows_of = [&](const Item& it, int& wy, int& wz) {
    if (EPI == MOE_EPI_SWIGLU) {
      wy = it.rtile * (ROWS / 2);
      wz = 2 * it.expert;
    } else {
      wy = 0;
      wz = it.expert * (N / (ROWS / 2)) + 2 * it.rtile;
    }
  };
  auto issue_weights = [&](uint32_t sb, uint32_t full, int s, int wy, int wz, int nr8) {
    mbar_arrive_expect_tx(full, kWBytes + LY::kA + nr8 * 4 * XBOX);
    tma_load_3d(sb, &wmap, full, s * SB, wy, wz);
    if (FMT == kFmtNF4) tma_load_3d(sb + kWBytes + kXBytes, &amap, full, s * 4, wy, wz);
  };
  // the stage's four 64-k blocks of the routed rows in one 3-D box
  auto issue_rows = [&](uint32_t sb, uint32_t full, int s, int start, int nr8) {
    tma_load_3d(sb + kWBytes, nr8 > 1 ? &xmap16 : &xmap8, full, 0, start, s * (SK / kBlock));
  };

  if (warp == PWARP) {
    // Set-up: the barriers, then (after the previous kernel unless chained)
    // the item list, then the first round of every ring, while the consumer
    // warps build the decode table.
    if (lane == 0) {
      for (int s = 0; s < NSLOTS; ++s) {
        mbar_init(smem_u32(&ms.full[s]), 1);
        mbar_init(smem_u32(&ms.empty[s]), CWARPS);
      }
      ms.abort_flag = 0;
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (!chain) {  // nothing is read or written before the previous kernel is done
      pdl_wait();
      pdl_trigger();
    }
    // item_prefix[e] = sum over e' < e of ceil(count / TOK) * rtiles
    bool bad = offsets[0] != 0 || offsets[E] != M_total;
    int run = 0;
    for (int b0 = 0; b0 < E; b0 += 32) {
      const int e = b0 + lane;
      int c = 0;
      if (e < E) {
        const int o0 = offsets[e], o1 = offsets[e + 1];
        ms.off[e] = o0;
        c = o1 - o0;
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
      ms.off[E] = offsets[E];
      ms.item_prefix[E] = run;
      ms.nitems = bad ? 0 : run;
      if (bad) set_dev_err(dev_err, MOE_DEVERR_BAD_OFFSETS);
    }
    __syncwarp();
    if (lane == 0) {
      // The first round of each ring.  Chain mode: only the weights (and
      // absmax), requested before the previous kernel (which writes A) has
      // finished; their barriers already expect the activation bytes too.
      const int total = ms.nitems;
#pragma unroll
      for (int g = 0; g < GROUPS; ++g) {
        int pre = 0;
        for (int i = blockIdx.x + g * gridDim.x; i < total && pre < ring_size(g); i += step) {
          const Item it = item_info(ms, E, rtiles, i);
          int wy, wz;
          rows_of(it, wy, wz);
          const int nr8 = (it.cnt + 7) / 8;
          for (int s = 0; s < KS && pre < ring_size(g); ++s, ++pre) {
            const int slot = ring_base(g) + pre;
            const uint32_t sb = LY::slot_addr(slot), full = smem_u32(&ms.full[slot]);
            issue_weights(sb, full, s, wy, wz, nr8);
            if (!chain) issue_rows(sb, full, s, it.start, nr8);
          }
        }
        ms.pre[g] = pre;
      }
      if (chain) {
        pdl_wait();
        pdl_trigger();
      }
    }
  } else {
    // byte b -> its two weights as an fp16 pair, the lower k in the low half:
    // NF4 {L[b >> 4], L[b & 15]}, INT4 {1024 + (b >> 4), 1024 + (b & 15)}
    // (0x6400 is fp16 1024, whose mantissa then holds the code).  One 256-byte
    // row per byte value, lane l's copy at 4 l (the upper 128 bytes of each
    // row are unused).  MXFP4 needs no table.
    for (int i = threadIdx.x; FMT != kFmtMXFP4 && i < 256 * 32; i += PWARP * 32) {
      const uint32_t b = (uint32_t)(i >> 5), l = (uint32_t)(i & 31);
      uint32_t v;
      if (FMT == kFmtNF4) {
        const __half2 h = __halves2half2(__float2half_rn(c_levels_dec[b >> 4]),
                                         __float2half_rn(c_levels_dec[b & 15]));
        v = *reinterpret_cast<const uint32_t*>(&h);
      } else {
        v = (0x6400u | (b >> 4)) | ((0x6400u | (b & 15u)) << 16);
      }
      lut[b * 64 + l] = v;
    }
  }
  __syncthreads();
  const int total = ms.nitems;

  if (warp == PWARP) {
    // ---------------- producer
    if (lane == 0) {
      // One cursor per group (item, stage of the item, ring position); the
      // loop serves whichever group's next slot is free.
      int ci[GROUPS], cs[GROUPS], cgi[GROUPS], cst[GROUPS], cwy[GROUPS], cwz[GROUPS],
          cnr[GROUPS], cstart[GROUPS], pre[GROUPS];
      uint32_t cph[GROUPS];
      auto load_item = [&](int g, int i) {
        const Item it = item_info(ms, E, rtiles, i);
        rows_of(it, cwy[g], cwz[g]);
        cnr[g] = (it.cnt + 7) / 8;
        cstart[g] = it.start;
      };
      int live = 0;
#pragma unroll
      for (int g = 0; g < GROUPS; ++g) {
        ci[g] = blockIdx.x + g * gridDim.x;
        cs[g] = cgi[g] = cst[g] = 0;
        cph[g] = 0;
        pre[g] = ms.pre[g];
        if (ci[g] < total) { load_item(g, ci[g]); ++live; }
      }
      uint32_t idle = 0;
      while (live > 0) {
        bool moved = false;
#pragma unroll
        for (int g = 0; g < GROUPS; ++g) {
          if (ci[g] >= total) continue;
          const int slot = ring_base(g) + cst[g];
          const uint32_t full = smem_u32(&ms.full[slot]);
          const uint32_t sb = LY::slot_addr(slot);
          // stages cgi < pre are the ring's first round, issued during the
          // set-up (in chain mode without their activation rows)
          const bool fresh = cgi[g] >= pre[g];
          if (fresh) {
            if (!mbar_test_wait(smem_u32(&ms.empty[slot]), cph[g] ^ 1)) continue;
            issue_weights(sb, full, cs[g], cwy[g], cwz[g], cnr[g]);
          }
          if (fresh || chain) issue_rows(sb, full, cs[g], cstart[g], cnr[g]);
          moved = true;
          ++cgi[g];
          if (++cst[g] == ring_size(g)) { cst[g] = 0; cph[g] ^= 1; }
          if (++cs[g] == KS) {
            cs[g] = 0;
            ci[g] += step;
            if (ci[g] < total) load_item(g, ci[g]); else --live;
          }
        }
        if (moved) {
          idle = 0;
        } else if (*reinterpret_cast<volatile int*>(&ms.abort_flag)) {
          break;
        } else if (++idle >= kSpinLimit) {
          *reinterpret_cast<volatile int*>(&ms.abort_flag) = 1;
          set_dev_err(dev_err, MOE_DEVERR_TIMEOUT);
          break;
        }
      }
    }
  } else {
    // ---------------- consumers
    const int g = warp / CWARPS;
    int stage = 0;
    uint32_t phase = 0;
    for (int i = blockIdx.x + g * gridDim.x; i < total; i += GROUPS * gridDim.x) {
      const Item it = item_info(ms, E, rtiles, i);
      bool ok;
      if (it.cnt > 8)
        ok = consume_item<FMT, EPI, OutT, 2>(ms, it, N, K, gscales, out, dev_err, warp % CWARPS,
                                             ring_base(g), ring_size(g), stage, phase);
      else
        ok = consume_item<FMT, EPI, OutT, 1>(ms, it, N, K, gscales, out, dev_err, warp % CWARPS,
                                             ring_base(g), ring_size(g), stage, phase);
      if (!ok) break;
    }
  }
  __syncwarp();  // the producer lane rejoins its warp before the CTA barrier
  __syncthreads();
}

int sm_count() { return device_sm_count(); }

template <int FMT, int EPI, typename OutT>
cudaError_t launch(const void* A, int A_rows, const uint8_t* packed, const void* scales,
                   const int32_t* offsets, int E, int N, int K, int M_total, void* out,
                   int32_t* dev_err, cudaStream_t s, bool chain) {
  using LY = Layout<FMT>;
  if (!tensor_map_encoder()) return cudaErrorNotSupported;
  const auto enc = encode_tiled_cached;
  CUtensorMap wmap, amap, xmap8, xmap16;
  const cuuint32_t estr[3] = {1, 1, 1};
  // Weight rows as [z][y][k]: SwiGLU z = 2e + half (gate / up), y = row in
  // the half; plain z = 64-row group, y = row in the group.  One box of
  // 2 x 64 rows is an item's 128 rows for one stage.
  const cuuint64_t ry = (EPI == MOE_EPI_SWIGLU) ? (cuuint64_t)N / 2 : (cuuint64_t)ROWS / 2;
  const cuuint64_t rz = (cuuint64_t)E * N / ry;
  {
    const cuuint64_t dims[3] = {(cuuint64_t)K / 2, ry, rz};
    const cuuint64_t strides[2] = {(cuuint64_t)K / 2, ry * (K / 2)};
    const cuuint32_t box[3] = {SB, ROWS / 2, 2};
    if (enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(packed), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  if (FMT == kFmtNF4) {
    // the absmax of the same rows, 4 blocks (one stage) per row; the L2
    // fetches whole 128-byte lines, so later stages of a row hit in L2
    const cuuint64_t dims[3] = {(cuuint64_t)K / kBlock, ry, rz};
    const cuuint64_t strides[2] = {(cuuint64_t)K / kBlock * 4, ry * (K / kBlock) * 4};
    const cuuint32_t box[3] = {SK / kBlock, ROWS / 2, 2};
    if (enc(&amap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
            const_cast<float*>(static_cast<const float*>(scales)), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    amap = wmap;  // unused
  }
  for (int rows : {8, 16}) {
    // routed activation rows as [K/64 blocks][rows][64 k]: one box of 4
    // blocks x 8 or 16 rows x 64 k is a stage's activations, laid out block
    // after block (8 or 16 swizzled 128-byte rows each)
    const cuuint64_t dims[3] = {(cuuint64_t)kBlock, (cuuint64_t)A_rows, (cuuint64_t)K / kBlock};
    const cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)kBlock * 2};
    const cuuint32_t box[3] = {kBlock, (cuuint32_t)rows, SK / kBlock};
    if (enc(rows == 8 ? &xmap8 : &xmap16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
            const_cast<void*>(A), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const size_t smem = LY::kEnd;  // absolute layout; the window starts at or below 1 KB
  auto kern = decode_kernel<FMT, EPI, OutT>;
  cudaError_t err = set_max_dynamic_smem_once(reinterpret_cast<const void*>(kern), (int)smem);
  if (err != cudaSuccess) return err;
  const int64_t max_items = ((int64_t)M_total / TOK + E) * (N / ROWS);
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(sm_count(), max_items));
  return launch_pdl(kern, dim3(grid), dim3(THREADS), smem, s, wmap, amap, xmap8, xmap16, scales,
                    offsets, E, N, K, M_total, reinterpret_cast<OutT*>(out), dev_err,
                    chain ? 1 : 0);
}

template <int FMT, int EPI>
cudaError_t launch_out(const void* A, int A_rows, const uint8_t* packed, const void* scales,
                       const int32_t* offsets, int E, int N, int K, int M_total, void* out,
                       moe_dtype_t out_dt, int32_t* dev_err, cudaStream_t s, bool chain) {
  if (out_dt == MOE_DT_F32)
    return launch<FMT, EPI, float>(A, A_rows, packed, scales, offsets, E, N, K, M_total, out,
                                   dev_err, s, chain);
  if (out_dt == MOE_DT_F16)
    return launch<FMT, EPI, __half>(A, A_rows, packed, scales, offsets, E, N, K, M_total, out,
                                    dev_err, s, chain);
  return launch<FMT, EPI, __nv_bfloat16>(A, A_rows, packed, scales, offsets, E, N, K, M_total,
                                         out, dev_err, s, chain);
}

template <int FMT>
cudaError_t launch_fmt(const void* A, int A_rows, const uint8_t* packed, const void* scales,
                       const int32_t* offsets, int E, int N, int K, int M_total,
                       moe_epilogue_t epi, void* out, moe_dtype_t out_dt, int32_t* dev_err,
                       cudaStream_t s, bool chain) {
  return epi == MOE_EPI_SWIGLU
             ? launch_out<FMT, MOE_EPI_SWIGLU>(A, A_rows, packed, scales, offsets, E, N, K,
                                               M_total, out, out_dt, dev_err, s, chain)
             : launch_out<FMT, MOE_EPI_NONE>(A, A_rows, packed, scales, offsets, E, N, K, M_total,
                                             out, out_dt, dev_err, s, chain);
}

}  // namespace dec
}  // namespace moe

namespace moe_launch {

bool grouped_gemm_decode_supported(int N, int K) {
  // absmax rows must be a multiple of 16 bytes for the TMA map: K % 256.
  return N % moe::dec::kNAlign == 0 && K % moe::dec::SK == 0;
}

// Activations must be fp16 rows in permuted order (no gather).
cudaError_t grouped_gemm_decode(const void* A, int A_rows, const uint8_t* packed,
                                const float* absmax, const int32_t* offsets, int E, int N, int K,
                                int M_total, moe_epilogue_t epi, void* out, moe_dtype_t out_dt,
                                int32_t* dev_err, cudaStream_t s, bool chain) {
  return moe::dec::launch_fmt<moe::kFmtNF4>(A, A_rows, packed, absmax, offsets, E, N, K, M_total,
                                            epi, out, out_dt, dev_err, s, chain);
}

bool grouped_gemm_int4_supported(int N, int K) {
  return N % moe::dec::kNAlign == 0 && K % moe::dec::SK == 0;
}

cudaError_t grouped_gemm_int4(const void* A, int A_rows, const uint8_t* packed,
                              const uint32_t* meta, const int32_t* offsets, int E, int N, int K,
                              int M_total, moe_epilogue_t epi, void* out, moe_dtype_t out_dt,
                              int32_t* dev_err, cudaStream_t s) {
  return moe::dec::launch_fmt<moe::kFmtINT4>(A, A_rows, packed, meta, offsets, E, N, K, M_total,
                                             epi, out, out_dt, dev_err, s, false);
}

bool grouped_gemm_mxfp4_supported(int N, int K) {
  return N % moe::dec::kNAlign == 0 && K % moe::dec::SK == 0;
}

cudaError_t grouped_gemm_mxfp4(const void* A, int A_rows, const uint8_t* packed,
                               const uint8_t* scales, const int32_t* offsets, int E, int N, int K,
                               int M_total, moe_epilogue_t epi, void* out, moe_dtype_t out_dt,
                               int32_t* dev_err, cudaStream_t s) {
  return moe::dec::launch_fmt<moe::kFmtMXFP4>(A, A_rows, packed, scales, offsets, E, N, K,
                                              M_total, epi, out, out_dt, dev_err, s, false);
}

}  // namespace moe_launch
