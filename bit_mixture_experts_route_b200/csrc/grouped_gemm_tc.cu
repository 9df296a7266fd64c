// Grouped NF4 GEMM, prefill path: tcgen05 tensor cores, weights decoded
// straight into tensor memory.
//
// "grouped-nf4-gemm & experts-4bit" (jordananderson-pages.pages.dev), first
// bullet: one launch for all active experts, the codebook decoded inside the
// GEMM, no dequantized copy of the weights in memory.  At prefill sizes
// (hundreds of routed rows per expert) the work is a dense contraction, so
// this kernel runs it on the 5th-generation tensor cores.
//
// Orientation: the MMA's M side is 128 weight rows (A, decoded NF4), its N
// side up to 256 routed rows of activations (B, fp16, from shared memory), so
// each decoded weight feeds up to 512 FLOP.  A never touches shared memory:
// decoder threads write it into tensor memory (tcgen05.st, one thread per
// weight row = TMEM lane) and the MMA reads it from there
// (tcgen05.mma ... [d], [a], b_desc).  Tensor memory (512 columns) holds the
// fp32 accumulator D = A * B^T (128 lanes x 256 columns) and an 8-slot ring of
// decoded 64-k weight stages (32 columns each, fp16 pairs).
//
// Persistent CTAs walk a tile list built on the device from expert_offsets
// (expert-major, then token tile, then weight-row tile), so no host sync is
// needed.  The CTA's k-stages, numbered S = 0, 1, 2, ... across its tiles,
// flow through three rings: activations (3 x 32 KB shared), packed NF4 rows
// (8 x 4 KB shared) and decoded weights (8 TMEM slots).  Waiting threads
// sleep in the barrier unit rather than spin.  Warp roles (864 threads):
//   warp 0      TMA producer: activation tiles [256 rows x 64 k] (128-byte
//               swizzle)
//   warp 1      TMEM allocator and MMA issuer (one thread): 4 x K16 per stage
//   warp 2      TMA producer: the tile's packed NF4 rows [128 rows x 32 B]
//   warps 3-18  decoders: four groups of four warps (one per TMEM lane
//               quarter); group g decodes the stages S = g (mod 4), so four
//               stages are decoded at once.  A thread turns its row's 32
//               packed bytes into 64 fp16 weights through a per-lane shared
//               table (byte -> {L[hi], L[lo]}), scales them by fp16(absmax)
//               (fetched one stage ahead) and stores them with tcgen05.st.
//   warps 19-26 epilogue: two warps per TMEM lane quarter, each taking
//               alternate 32-column blocks: tcgen05.ld, SwiGLU (gate and up
//               rows interleaved in the tile, paired with one shuffle per two
//               tokens) or a plain copy, a transpose through shared memory and
//               16-byte row stores.  A warp releases the accumulator right
//               after its last tcgen05.ld of the tile.
// Every mbarrier wait is bounded; on expiry the kernel sets
// MOE_DEVERR_TIMEOUT, every role leaves its loop, TMEM is freed and the
// kernel returns.
#include "common.cuh"

namespace moe {
namespace tc {

constexpr int BM = 128;          // weight rows per tile (MMA M)
constexpr int BN = 256;          // routed rows per tile (max MMA N)
constexpr int BK = 64;           // k per stage = one NF4 block
constexpr int BSTAGES = 3;       // activation ring
constexpr int B_STAGE = BN * BK * 2;   // 32 KB
constexpr int B_BOX_ROWS = 128;        // TMA box: 64 k x 128 rows
constexpr int RAW_RING = 8;            // packed-row ring (shared memory)
constexpr int RING = 8;                // decoded-weight ring (tensor memory)
constexpr int RAW_STAGE = BM * BK / 2; // 4 KB
constexpr int GROUPS = 4;              // decoder groups (stages in flight)
constexpr int DEC_WARPS = 4 * GROUPS;
constexpr int W_BPROD = 0, W_MMA = 1, W_RPROD = 2, W_DEC = 3, W_EPI = W_DEC + DEC_WARPS;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 32 * (W_EPI + EPI_WARPS);
constexpr int TMEM_COLS = 512;
constexpr int ACC_COL = 0;             // accumulator: columns [0, 256)
constexpr int A_COL = BN;              // decoded-weight slot a: columns 256 + 32 a
constexpr int A_SLOT_COLS = BK / 2;
constexpr int STG_BYTES = 32 * 32 * 4; // epilogue transpose buffer per warp
constexpr uint32_t kWaitLimit = 1u << 20;  // suspended tries before a wait gives up
constexpr uint32_t kSuspendNs = 1000;       // longest sleep of one try
static_assert(A_COL + RING * A_SLOT_COLS <= TMEM_COLS, "tensor memory budget");
static_assert(BSTAGES * B_STAGE + RAW_RING * RAW_STAGE + EPI_WARPS * STG_BYTES + 256 * 32 * 4 +
                      2 * 1025 * 4 + 1024 <
                  227 * 1024,
              "shared memory budget");
static_assert(BSTAGES < RING, "activation slots are released through the TMEM-slot barriers");
static_assert(RING % GROUPS == 0 && RAW_RING % GROUPS == 0,
              "a group always meets its own slots");

struct __align__(8) Smem {
  uint8_t b[BSTAGES][B_STAGE];  // 1024-aligned (struct placed at 1024)
  uint8_t raw[RAW_RING][RAW_STAGE];
  uint8_t stg[EPI_WARPS][STG_BYTES];
  uint32_t lut[256 * 32];
  uint64_t raw_full[RAW_RING], raw_empty[RAW_RING];
  // ready[s]: stage s's decoded weights (four decoder-warp arrivals) and its
  // activation tile (producer arrival + TMA bytes); a_empty[s]: its MMAs done
  uint64_t ready[RING], a_empty[RING];
  uint64_t acc_full, acc_empty;
  uint32_t tmem_base;
  int abort_flag;
  int ntiles_total;
  int tile_prefix[1025];
  int off[1025];  // expert_offsets, copied once
};

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
// Same, but the thread may sleep in the barrier unit up to kSuspendNs until
// the phase completes, instead of re-issuing: waiting warps leave the issue
// slots to the warps that have work.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}

// Bounded wait: false (and the abort flag set) if the phase never completes
// (kWaitLimit suspended tries, well under a second each way) or another role
// already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, Smem& sm,
                                          int32_t* dev_err) {
  if (mbar_try_wait(bar, parity)) return true;
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait_suspend(bar, parity)) return true;
    if (*reinterpret_cast<volatile int*>(&sm.abort_flag)) return false;
  }
  *reinterpret_cast<volatile int*>(&sm.abort_flag) = 1;
  set_dev_err(dev_err, MOE_DEVERR_TIMEOUT);
  return false;
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), sm_100 descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;               // LBO (unused for swizzled K-major)
  d |= (uint64_t)(1024u >> 4) << 32;     // SBO
  d |= (uint64_t)1u << 46;               // version
  d |= (uint64_t)2u << 61;               // SWIZZLE_128B
  return d;
}

// Instruction descriptor: D fp32, A/B fp16, both K-major, M = 128, N = n.
__device__ __forceinline__ uint32_t idesc_f16(int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
        "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
        "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}


// Decoded weights into tensor memory: 16 consecutive 32-bit columns of this
// thread's lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// D (TMEM) += A (TMEM) * B (shared memory descriptor)
__device__ __forceinline__ void mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ uint4 lds128(const void* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_u32(p)));
  return v;
}

__constant__ float c_levels_tc[16] = {MOE_NF4_LEVEL_LIST};

// Tile t's expert and weight-row tile: expert e with
// tile_prefix[e] <= t < tile_prefix[e+1] (shared memory only).
struct TileId {
  int expert, ntile, ttile;
};
__device__ __forceinline__ TileId tile_id(const Smem& sm, int E, int n_tiles, int t) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (sm.tile_prefix[mid] <= t) lo = mid; else hi = mid;
  }
  const int local = t - sm.tile_prefix[lo];
  const int tt = local / n_tiles;
  return TileId{lo, local - tt * n_tiles, tt};
}

struct TileInfo {
  int expert, row0, nrows, ntile;
};
__device__ __forceinline__ TileInfo tile_info(const Smem& sm, int E, int n_tiles, int t) {
  const TileId id = tile_id(sm, E, n_tiles, t);
  TileInfo ti;
  ti.expert = id.expert;
  ti.ntile = id.ntile;
  ti.row0 = sm.off[id.expert] + id.ttile * BN;
  ti.nrows = min(BN, sm.off[id.expert + 1] - ti.row0);
  return ti;
}

// A thread's scales of one 64-k stage of its weight row as fp16 pairs for the
// two 32-element halves: NF4 one fp32 absmax (both halves; `bad` when its
// fp16 is subnormal or not finite), MXFP4 two E8M0 bytes (`bad` outside the
// range where every scaled value is exact in fp16).
template <int FMT>
__device__ __forceinline__ void stage_scales(uint32_t sc, uint32_t& h0, uint32_t& h1, bool& bad) {
  if (FMT == kFmtNF4) {
    const float a = __uint_as_float(sc);
    bad |= a != 0.0f && !(a >= 6.103515625e-05f && a <= 65504.0f);
    const __half2 ah = __float2half2_rn(a);
    h0 = h1 = *reinterpret_cast<const uint32_t*>(&ah);
  } else {
    h0 = mx_scale_h2(sc & 0xFFu, bad);
    h1 = mx_scale_h2((sc >> 8) & 0xFFu, bad);
  }
}

template <int FMT, int EPI, typename OutT>
__global__ void __launch_bounds__(THREADS, 1) nf4_tc_kernel(
    const __grid_constant__ CUtensorMap bmap, const __grid_constant__ CUtensorMap wmap,
    const void* __restrict__ scales, const int32_t* __restrict__ offsets, int E, int N, int K,
    int M_total, OutT* __restrict__ out, int32_t* dev_err, int chain) {
  extern __shared__ uint8_t smem_raw[];
  if (!chain) {  // nothing is read or written before the previous kernel is done
    pdl_wait();
    pdl_trigger();
  }
  Smem& sm = *reinterpret_cast<Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = N / BM;
  const int KT = K / BK;

  // ---- setup: barriers, offsets, decode table, tile list, TMEM
  if (threadIdx.x == 0) {
    for (int s = 0; s < BSTAGES; ++s) {
    }
    for (int s = 0; s < RAW_RING; ++s) {
      mbar_init(&sm.raw_full[s], 1);
      mbar_init(&sm.raw_empty[s], 4);   // the four warps of the decoding group
    }
    for (int s = 0; s < RING; ++s) {
      mbar_init(&sm.ready[s], 4 + 1);
      mbar_init(&sm.a_empty[s], 1);     // MMA completion (tcgen05.commit)
    }
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.acc_empty, 32 * EPI_WARPS);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int e = threadIdx.x; e <= E; e += THREADS) sm.off[e] = offsets[e];
  // byte -> its two weights as an fp16 pair, the lower k in the low half:
  // NF4 {L[high nibble], L[low nibble]}, MXFP4 {e2m1(low), e2m1(high)}
  for (int i = threadIdx.x; i < 256 * 32; i += THREADS) {
    const int b = i >> 5;
    if (FMT == kFmtNF4) {
      const __half2 h = __halves2half2(__float2half_rn(c_levels_tc[b >> 4]),
                                       __float2half_rn(c_levels_tc[b & 15]));
      sm.lut[i] = *reinterpret_cast<const uint32_t*>(&h);
    } else {
      sm.lut[i] = e2m1_h((uint32_t)b & 15u) | (e2m1_h((uint32_t)b >> 4) << 16);
    }
  }
  if (warp == W_MMA) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&sm.tmem_base)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  __syncthreads();
  if (warp == W_BPROD) {
    // tile_prefix[e] = sum over e' < e of ceil(count / BN) * n_tiles
    bool bad = sm.off[0] != 0 || sm.off[E] != M_total;
    int run = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int c = 0;
      if (e < E) {
        c = sm.off[e + 1] - sm.off[e];
        if (c < 0) { bad = true; c = 0; }
      }
      int tiles = ((c + BN - 1) / BN) * n_tiles;
      int incl = tiles;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (e < E) sm.tile_prefix[e] = run + incl - tiles;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      sm.tile_prefix[E] = run;
      sm.ntiles_total = bad ? 0 : run;
      if (bad) set_dev_err(dev_err, MOE_DEVERR_BAD_OFFSETS);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sm.tmem_base;
  const int total = sm.ntiles_total;

  if (warp == W_BPROD) {
    // ---------------- TMA producer: activation tiles, stage S of the CTA
    if (lane == 0) {
      // chain mode: the previous kernel writes A; the weight producer and the
      // decoders started without waiting for it
      if (chain) {
        pdl_wait();
        pdl_trigger();
      }
      // slot S mod BSTAGES is free once the MMAs of stage S - BSTAGES are
      // done; their completion is the a_empty barrier of that stage's TMEM
      // slot (one commit per stage serves both rings)
      int bs = 0, S = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const TileInfo ti = tile_info(sm, E, n_tiles, t);
        const int nmma = (ti.nrows + 15) & ~15;
        const int boxes = (nmma + B_BOX_ROWS - 1) / B_BOX_ROWS;
        for (int ks = 0; ks < KT; ++ks, ++S) {
          if (S >= BSTAGES) {
            const int P = S - BSTAGES;
            if (!(ok = mbar_wait(&sm.a_empty[P % RING], (uint32_t)(P / RING) & 1u, sm, dev_err)))
              break;
          }
          uint64_t* rdy = &sm.ready[S % RING];
          mbar_arrive_expect_tx(rdy, boxes * B_BOX_ROWS * BK * 2);
          for (int b = 0; b < boxes; ++b)
            tma_load_2d(sm.b[bs] + b * (B_BOX_ROWS * BK * 2), &bmap, rdy, ks * BK,
                        ti.row0 + b * B_BOX_ROWS);
          if (++bs == BSTAGES) bs = 0;
        }
      }
    }
  } else if (warp == W_MMA) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint64_t bdesc0 = sw128_desc(smem_u32(sm.b[0]));
      int bs = 0, as = 0;
      uint32_t aph = 0;
      bool ok = true;
      int lt = 0;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++lt) {
        const TileInfo ti = tile_info(sm, E, n_tiles, t);
        const int nmma = (ti.nrows + 15) & ~15;
        // the single accumulator must have been drained by the epilogue
        if (!(ok = mbar_wait(&sm.acc_empty, (lt & 1) ^ 1, sm, dev_err))) break;
        tc_fence_after();
        const uint32_t idesc = idesc_f16(nmma);
        const uint32_t dcol = tmem_base + ACC_COL;
        for (int ks = 0; ks < KT; ++ks) {
          if (!(ok = mbar_wait(&sm.ready[as], aph, sm, dev_err))) break;
          tc_fence_after();
          // K slice kk: 8 more TMEM columns of A; 32 bytes further into the
          // swizzled activation rows (+2 in the descriptor's address field)
          const uint32_t acol = tmem_base + A_COL + as * A_SLOT_COLS;
          const uint64_t bd = bdesc0 + (uint64_t)(bs * (B_STAGE >> 4));
          mma_ts(dcol, acol, bd, idesc, ks != 0);
          mma_ts(dcol, acol + 8, bd + 2, idesc, 1u);
          mma_ts(dcol, acol + 16, bd + 4, idesc, 1u);
          mma_ts(dcol, acol + 24, bd + 6, idesc, 1u);
          mma_commit(&sm.a_empty[as]);  // frees TMEM slot as and activation slot bs
          if (++bs == BSTAGES) bs = 0;
          if (++as == RING) { as = 0; aph ^= 1; }
        }
        if (ok) mma_commit(&sm.acc_full);
      }
    }
  } else if (warp == W_RPROD) {
    // ---------------- TMA producer: packed NF4 rows of the tile
    if (lane == 0) {
      int rs = 0;
      uint32_t rph = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const TileId id = tile_id(sm, E, n_tiles, t);
        int y0, y1;  // first weight row of each 64-row box
        if (EPI == MOE_EPI_SWIGLU) {
          y0 = id.expert * N + id.ntile * (BM / 2);  // gate rows
          y1 = y0 + N / 2;                           // matching up rows
        } else {
          y0 = id.expert * N + id.ntile * BM;
          y1 = y0 + BM / 2;
        }
        for (int ks = 0; ks < KT; ++ks) {
          if (!(ok = mbar_wait(&sm.raw_empty[rs], rph ^ 1, sm, dev_err))) break;
          mbar_arrive_expect_tx(&sm.raw_full[rs], RAW_STAGE);
          tma_load_2d(sm.raw[rs], &wmap, &sm.raw_full[rs], ks * (BK / 2), y0);
          tma_load_2d(sm.raw[rs] + (BM / 2) * (BK / 2), &wmap, &sm.raw_full[rs], ks * (BK / 2), y1);
          if (++rs == RAW_RING) { rs = 0; rph ^= 1; }
        }
      }
    }
  } else if (warp < W_EPI) {
    // ---------------- decoders: group g, TMEM lane quarter q, tile row m
    const int g = (warp - W_DEC) >> 2;
    const int q = warp & 3;
    const int m = 32 * q + lane;
    // row of the raw tile holding tile row m (SwiGLU tiles interleave gate
    // and up rows: even m = gate j, odd m = up j; the raw tile holds the 64
    // gate rows, then the 64 up rows)
    const int rrow = (EPI == MOE_EPI_SWIGLU) ? ((m & 1) ? BM / 2 + (m >> 1) : (m >> 1)) : m;
    const uint32_t* lut = sm.lut + lane;
    const uint32_t tlane = tmem_base + ((uint32_t)(32 * q) << 16);
    // scales of this thread's weight row in tile t (null past the CTA's last
    // tile), stage ks at word ks: NF4 the fp32 absmax of block ks, MXFP4 the
    // two E8M0 bytes of the stage; walked one own stage ahead without
    // divisions
    auto row_scales = [&](int t) -> const uint8_t* {
      if (t >= total) return nullptr;
      const TileId id = tile_id(sm, E, n_tiles, t);
      int row;
      if (EPI == MOE_EPI_SWIGLU) {
        const int j = id.ntile * (BM / 2) + (m >> 1);
        row = (m & 1) ? (N / 2 + j) : j;
      } else {
        row = id.ntile * BM + m;
      }
      const size_t r = (size_t)id.expert * N + row;
      return reinterpret_cast<const uint8_t*>(scales) +
             (FMT == kFmtNF4 ? r * (size_t)KT * 4 : r * (size_t)(K / 32));
    };
    auto fetch = [&](const uint8_t* row, int ks) -> uint32_t {
      if (FMT == kFmtNF4) return __ldg(reinterpret_cast<const uint32_t*>(row) + ks);
      return __ldg(reinterpret_cast<const uint16_t*>(row) + ks);
    };
    int n_ks = g, n_t = blockIdx.x;
    while (n_ks >= KT) { n_ks -= KT; n_t += gridDim.x; }
    const uint8_t* n_row = row_scales(n_t);
    uint32_t sc_cur = n_row ? fetch(n_row, n_ks) : 0u;
    bool have = n_row != nullptr;
    bool bad_scale = false;  // a scale the fp16 weights cannot carry exactly
    for (int S = g; have; S += GROUPS) {
      const int slot = S % RING, rslot = S % RAW_RING;
      const uint32_t ph = (uint32_t)(S / RING) & 1u, rph = (uint32_t)(S / RAW_RING) & 1u;
      n_ks += GROUPS;
      while (n_ks >= KT && n_row) {
        n_ks -= KT;
        n_t += gridDim.x;
        n_row = row_scales(n_t);
      }
      const bool have_next = n_row != nullptr;
      const uint32_t sc_next = have_next ? fetch(n_row, n_ks) : 0u;  // one stage ahead
      // warp-uniform outcomes: tcgen05.st below is .aligned
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.raw_full[rslot], rph, sm, dev_err))) break;
      const uint8_t* rp = sm.raw[rslot] + rrow * (BK / 2);
      const uint4 w0 = lds128(rp), w1 = lds128(rp + 16);
      uint32_t sh[2];
      stage_scales<FMT>(sc_cur, sh[0], sh[1], bad_scale);
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.a_empty[slot], ph ^ 1, sm, dev_err))) break;
      tc_fence_after();
      const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const __half2 ah = *reinterpret_cast<const __half2*>(&sh[half]);
        uint32_t hv[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t w = words[4 * half + c];
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const uint32_t raw = lut[__byte_perm(w, 0, 0x4440u | b) << 5];
            __half2 v = __hmul2(*reinterpret_cast<const __half2*>(&raw), ah);
            hv[4 * c + b] = *reinterpret_cast<uint32_t*>(&v);
          }
        }
        tmem_st16(tlane + A_COL + slot * A_SLOT_COLS + 16 * half, hv);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sm.ready[slot]);
        mbar_arrive(&sm.raw_empty[rslot]);  // its bytes are decoded
      }
      sc_cur = sc_next;
      have = have_next;
    }
    // the loop exits are warp-uniform, so every lane takes part
    if (__any_sync(0xffffffffu, bad_scale) && lane == 0) set_dev_err(dev_err, MOE_DEVERR_RANGE);
  } else {
    // ---------------- epilogue: warp (q, hc) reads TMEM lanes 32q .. 32q+31,
    // columns of half hc of each 64-column block (two warps per lane quarter)
    const int ew = warp - W_EPI;
    const int q = warp & 3;       // consecutive warps cover every lane quarter
    const int hc = ew >> 2;       // which 32 of each 64 columns
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    uint8_t* stg = sm.stg[ew];
    // a staged row: 16 outputs (SwiGLU pairs) or 32 (plain) of one token
    constexpr int OUT_COLS = (EPI == MOE_EPI_SWIGLU) ? 16 : 32;
    constexpr int ROWB = OUT_COLS * (int)sizeof(OutT);
    constexpr int V = ROWB / 16;  // 16-byte pieces per staged row
    bool ok = true;
    bool ovf = false;  // an fp16 output that overflowed
    int lt = 0;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++lt) {
      const TileInfo ti = tile_info(sm, E, n_tiles, t);
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&sm.acc_full, lt & 1, sm, dev_err)))) break;
      tc_fence_after();
      const int ncols = (ti.nrows + 15) & ~15;
      // first output column of this warp's rows
      const int col0 = (EPI == MOE_EPI_SWIGLU) ? ti.ntile * (BM / 2) + 16 * q : ti.ntile * BM + 32 * q;
      const int ldo = (EPI == MOE_EPI_SWIGLU) ? N / 2 : N;
      bool released = false;
      for (int c0 = 32 * hc; c0 < ncols; c0 += 64) {
        uint32_t v[32];
        tmem_ld32(tmem_base + lane_addr + ACC_COL + c0, v);
        if (c0 + 64 >= ncols) {
          // this warp's last read of the accumulator: hand it back to the
          // MMA before the math and the stores
          tc_fence_before();
          mbar_arrive(&sm.acc_empty);
          released = true;
        }
        if (EPI == MOE_EPI_SWIGLU) {
          // lanes 2p (gate row) and 2p+1 (up row) of output column p: the
          // even lane finishes tokens [0,16), the odd lane [16,32); one
          // exchange per pair of tokens, no divergence
          const bool up = lane & 1;
          const int p = lane >> 1;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float lo = __uint_as_float(v[i]), hi = __uint_as_float(v[16 + i]);
            const float recv = __shfl_xor_sync(0xffffffffu, up ? lo : hi, 1);
            const float gt = up ? recv : lo, u = up ? hi : recv;
            // silu(g) * u with the fast exp and division intrinsics: their
            // relative error (~1e-6) is far below the fp16/bf16 output rounding
            const float h = __fdividef(gt, 1.0f + __expf(-gt)) * u;
            const int tok = (up ? 16 : 0) + i;
            ovf |= c0 + tok < ti.nrows && overflows_out<OutT>(h);
            reinterpret_cast<OutT*>(stg + tok * ROWB)[p] = from_f32<OutT>(h);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float y = __uint_as_float(v[i]);
            ovf |= c0 + i < ti.nrows && overflows_out<OutT>(y);
            reinterpret_cast<OutT*>(stg + i * ROWB)[lane] = from_f32<OutT>(y);
          }
        }
        __syncwarp();
        // staged rows -> global, 16 bytes per lane
#pragma unroll
        for (int idx = lane; idx < 32 * V; idx += 32) {
          const int tok = idx / V, piece = idx - tok * V;
          if (c0 + tok < ti.nrows) {
            const uint4 val = lds128(stg + tok * ROWB + piece * 16);
            *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(
                out + (size_t)(ti.row0 + c0 + tok) * ldo + col0) + piece * 16) = val;
          }
        }
        __syncwarp();
      }
      if (!released) {  // no columns for this warp in this tile
        tc_fence_before();
        mbar_arrive(&sm.acc_empty);
      }
    }
    // the loop exits are warp-uniform, so every lane takes part
    if (__any_sync(0xffffffffu, ovf) && lane == 0) set_dev_err(dev_err, MOE_DEVERR_RANGE);
  }

  // single-lane roles (producers, MMA issuer) rejoin their warp before the
  // CTA-wide barrier
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS));
  }
}

int sm_count() { return device_sm_count(); }

template <int FMT, int EPI, typename OutT>
cudaError_t launch(const void* A, const uint8_t* packed, const void* scales,
                   const int32_t* offsets, int E, int N, int K, int M_total, void* out,
                   int32_t* dev_err, cudaStream_t s, bool chain) {
  if (!tensor_map_encoder()) return cudaErrorNotSupported;
  const auto enc = encode_tiled_cached;
  CUtensorMap map, wmap;
  const cuuint32_t estr[2] = {1, 1};
  {
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M_total};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {BK, B_BOX_ROWS};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(A), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    // packed rows as a 2-D byte tensor [E*N, K/2]; box = 32 bytes x 64 rows
    const cuuint64_t dims[2] = {(cuuint64_t)K / 2, (cuuint64_t)E * N};
    const cuuint64_t strides[1] = {(cuuint64_t)K / 2};
    const cuuint32_t box[2] = {BK / 2, BM / 2};
    if (enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(packed), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const size_t smem = sizeof(Smem) + 1024;
  auto kern = nf4_tc_kernel<FMT, EPI, OutT>;
  cudaError_t err = set_max_dynamic_smem_once(reinterpret_cast<const void*>(kern), (int)smem);
  if (err != cudaSuccess) return err;
  // Upper bound on tiles: every expert's rows rounded up to BN, plus one
  // partial tile per expert; the kernel derives the exact list itself.
  const int64_t max_tiles = ((int64_t)M_total / BN + E) * (N / BM);
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(sm_count(), max_tiles));
  return launch_pdl(kern, dim3(grid), dim3(THREADS), smem, s, map, wmap, scales, offsets, E, N, K,
                    M_total, reinterpret_cast<OutT*>(out), dev_err, chain ? 1 : 0);
}

template <int FMT>
cudaError_t launch_fmt(const void* A, const uint8_t* packed, const void* scales,
                       const int32_t* offsets, int E, int N, int K, int M_total,
                       moe_epilogue_t epi, void* out, moe_dtype_t out_dt, int32_t* dev_err,
                       cudaStream_t s, bool chain) {
  if (epi == MOE_EPI_SWIGLU) {
    if (out_dt == MOE_DT_F16)
      return launch<FMT, MOE_EPI_SWIGLU, __half>(A, packed, scales, offsets, E, N, K, M_total,
                                                 out, dev_err, s, chain);
    if (out_dt == MOE_DT_BF16)
      return launch<FMT, MOE_EPI_SWIGLU, __nv_bfloat16>(A, packed, scales, offsets, E, N, K,
                                                        M_total, out, dev_err, s, chain);
    return launch<FMT, MOE_EPI_SWIGLU, float>(A, packed, scales, offsets, E, N, K, M_total, out,
                                              dev_err, s, chain);
  }
  if (out_dt == MOE_DT_F16)
    return launch<FMT, MOE_EPI_NONE, __half>(A, packed, scales, offsets, E, N, K, M_total, out,
                                             dev_err, s, chain);
  if (out_dt == MOE_DT_BF16)
    return launch<FMT, MOE_EPI_NONE, __nv_bfloat16>(A, packed, scales, offsets, E, N, K,
                                                    M_total, out, dev_err, s, chain);
  return launch<FMT, MOE_EPI_NONE, float>(A, packed, scales, offsets, E, N, K, M_total, out,
                                          dev_err, s, chain);
}

}  // namespace tc
}  // namespace moe

namespace moe_launch {

bool grouped_gemm_tc_supported(int N, int K, moe_epilogue_t epi) {
  (void)epi;
  return N % moe::tc::BM == 0 && K % moe::tc::BK == 0 && K >= moe::tc::BK;
}

cudaError_t grouped_gemm_tc(const void* A, moe_dtype_t a_dt, int A_rows, const int32_t* gather,
                            int k, const uint8_t* packed, const float* absmax,
                            const int32_t* offsets, int E, int N, int K, int M_total,
                            moe_epilogue_t epi, void* out, moe_dtype_t out_dt, int32_t* dev_err,
                            cudaStream_t s, bool chain) {
  (void)k;
  if (gather || a_dt != MOE_DT_F16 || A_rows < M_total) return cudaErrorNotSupported;
  return moe::tc::launch_fmt<moe::kFmtNF4>(A, packed, absmax, offsets, E, N, K, M_total, epi,
                                           out, out_dt, dev_err, s, chain);
}

cudaError_t grouped_gemm_tc_mxfp4(const void* A, int A_rows, const uint8_t* packed,
                                  const uint8_t* scales, const int32_t* offsets, int E, int N,
                                  int K, int M_total, moe_epilogue_t epi, void* out,
                                  moe_dtype_t out_dt, int32_t* dev_err, cudaStream_t s) {
  if (A_rows < M_total) return cudaErrorNotSupported;
  return moe::tc::launch_fmt<moe::kFmtMXFP4>(A, packed, scales, offsets, E, N, K, M_total, epi,
                                             out, out_dt, dev_err, s, false);
}

}  // namespace moe_launch
