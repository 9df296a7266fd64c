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
//   warp 0      TMA producer: activation tiles [the MMA's N rows x 64 k]
//               (128-byte swizzle), one box of exactly that height
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
//
// Pair form (PAIR = 2, used when N % 256 == 0): the CTAs run as clusters of
// two on two SMs and every tile is 256 weight rows.  Each CTA decodes its
// 128 rows into its own tensor memory and loads half of the tile's routed
// rows (B) into its own shared memory; the leader CTA (rank 0) issues
// tcgen05.mma.cta_group::2 with M = 256, which reads A and B from both CTAs
// and writes each CTA's 128 x N block of D into that CTA's tensor memory.
// One MMA instruction then does twice the work of the single-CTA form, and
// each routed-row tile crosses L2 -> SM once per 256 weight rows instead of
// per 128.  The peer's decoders and its B loads signal the leader's `ready`
// barriers directly (remote mbarrier arrive, and TMA with .cta_group::2);
// the leader's commits arrive on both CTAs' barriers (.multicast::cluster);
// the peer's epilogue hands the accumulator back with remote arrives.  No
// TMA load uses multicast.
#include <type_traits>

#include "common.cuh"

namespace moe {
namespace tc {

constexpr int BM = 128;          // weight rows per tile (MMA M)
constexpr int BN = 256;          // routed rows per tile (max MMA N)
constexpr int BK = 64;           // k per stage = one NF4 block
constexpr int B_STAGE = BN * BK * 2;   // 32 KB: a tile's routed rows (at most 256)
constexpr int B_MAPS = BN / 16;        // activation box heights 16, 32, ..., 256 rows

constexpr int RAW_RING = 8;            // packed-row ring (shared memory)
constexpr int RING = 8;                // decoded-weight ring (tensor memory)
constexpr int RAW_STAGE = BM * BK / 2; // 4 KB
// transposed (backward) form: 64 weight rows x 128 columns of packed bytes
// (4 KB) and their absmax, 4 fp32 per row (1 KB), per stage
constexpr int RAW_STAGE_T = RAW_STAGE + 64 * 16;
constexpr int EPI_SWIGLU_BWD = 2;       // transposed down GEMM + SwiGLU backward
constexpr int GROUPS = 4;              // decoder groups (stages in flight)
constexpr int DEC_WARPS = 4 * GROUPS;
constexpr int W_BPROD = 0, W_MMA = 1, W_RPROD = 2, W_DEC = 3, W_EPI = W_DEC + DEC_WARPS;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 32 * (W_EPI + EPI_WARPS);
constexpr int TMEM_COLS = 512;
constexpr int ACC_COL = 0;             // accumulator: columns [0, 256)
constexpr int A_COL = BN;              // decoded-weight slot a: columns 256 + 32 a
constexpr int A_SLOT_COLS = BK / 2;
constexpr int STG_BYTES = 32 * 32 * 4; // epilogue transpose buffer per warp (fp32 rows)
constexpr uint32_t kWaitLimit = 1u << 20;  // suspended tries before a wait gives up
constexpr uint32_t kSuspendNs = 1000;       // longest sleep of one try
static_assert(A_COL + RING * A_SLOT_COLS <= TMEM_COLS, "tensor memory budget");
static_assert(RING % GROUPS == 0 && RAW_RING % GROUPS == 0,
              "a group always meets its own slots");

// One tensor map of the activation (or gradient) rows per box height, 16 to
// 256 rows in steps of 16: a stage loads exactly the rows its MMAs read.
struct __align__(64) BMaps {
  CUtensorMap m[B_MAPS];
};

// Shared memory of one kernel form.  The activation producer can only run
// NBS stages ahead of the MMAs (it refills a stage's slot once that stage's
// MMAs are done), so a form takes as many 32-KB activation stages as its
// packed-row slots (RAWB: 4 KB, or 5 KB with the transposed form's absmax)
// and epilogue transpose buffers (STGB per warp: 32 rows of 32 outputs) leave
// room for: 4 for the forward form with 16-bit outputs, 3 otherwise.
template <int NBS, int RAWB, int STGB>
struct __align__(8) SmemT {
  static constexpr int kNBS = NBS;
  uint8_t b[NBS][B_STAGE];  // 1024-aligned (struct placed at 1024)
  uint8_t raw[RAW_RING][RAWB];
  uint8_t stg[EPI_WARPS][STGB];
  uint32_t lut[256 * 32];
  uint64_t raw_full[RAW_RING], raw_empty[RAW_RING];
  // ready[s]: stage s's decoded weights (four decoder-warp arrivals) and its
  // activation tile (producer arrival + TMA bytes); a_empty[s]: its MMAs done
  uint64_t ready[RING], a_empty[RING];
  uint64_t acc_full, acc_empty;
  uint64_t drain;  // pair form: the leader's MMAs all complete
  uint32_t tmem_base;
  int abort_flag;
  int ntiles_total;
  int tile_prefix[1025];
  int off[1025];  // expert_offsets, copied once
};
template <typename OutT, bool TR>
using SmemFor = typename std::conditional<(sizeof(OutT) == 2 && !TR), SmemT<4, RAW_STAGE, 2048>,
                                          SmemT<3, RAW_STAGE_T, STG_BYTES>>::type;
static_assert(sizeof(SmemT<4, RAW_STAGE, 2048>) + 1024 <= 227 * 1024, "shared memory budget");
static_assert(sizeof(SmemT<3, RAW_STAGE_T, STG_BYTES>) + 1024 <= 227 * 1024,
              "shared memory budget");
static_assert(4 < RING, "activation slots are released through the TMEM-slot barriers");

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

// The same two waits with acquire at cluster scope, for barriers that the
// other CTA of a pair arrives on.
__device__ __forceinline__ bool mbar_try_wait_cl(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_try_wait_suspend_cl(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}

// Non-blocking test of a phase (the MMA issuer polls with it: a thread woken
// from a suspended try_wait resumes later than one that polls).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
constexpr uint32_t kPollLimit = 1u << 26;  // polls before a polled wait gives up (~1 s)

// Bounded polled wait (see mbar_wait), for the single MMA-issuing thread.
template <class SM>
__device__ __forceinline__ bool mbar_poll(uint64_t* bar, uint32_t parity, SM& sm,
                                          int32_t* dev_err) {
  for (uint32_t i = 0; i < kPollLimit; ++i) {
    if (mbar_test_wait(bar, parity)) return true;
    if ((i & 255u) == 255u && *reinterpret_cast<volatile int*>(&sm.abort_flag)) return false;
  }
  *reinterpret_cast<volatile int*>(&sm.abort_flag) = 1;
  set_dev_err(dev_err, MOE_DEVERR_TIMEOUT);
  return false;
}

// Bounded wait: false (and the abort flag set) if the phase never completes
// (kWaitLimit suspended tries, well under a second each way) or another role
// already aborted.  CLUSTER: acquire at cluster scope.
template <bool CLUSTER = false, class SM>
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, SM& sm,
                                          int32_t* dev_err) {
  if (CLUSTER ? mbar_try_wait_cl(bar, parity) : mbar_try_wait(bar, parity)) return true;
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (CLUSTER ? mbar_try_wait_suspend_cl(bar, parity) : mbar_try_wait_suspend(bar, parity))
      return true;
    if (*reinterpret_cast<volatile int*>(&sm.abort_flag)) return false;
  }
  *reinterpret_cast<volatile int*>(&sm.abort_flag) = 1;
  set_dev_err(dev_err, MOE_DEVERR_TIMEOUT);
  return false;
}

// ---- pair form (clusters of two CTAs)
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The shared::cluster address of the same shared variable in CTA `rank`.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
               : "memory");
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// The same load issued for the pair: the destination is this CTA's shared
// memory, the barrier may be the other CTA's (a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map,
                                                 uint32_t cluster_bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(cluster_bar), "r"(x), "r"(y)
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

// Instruction descriptor: D fp32, A/B fp16, both K-major, M = m, N = n.
__device__ __forceinline__ uint32_t idesc_f16(int m, int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
// Pair form: the leader's MMAs so far done -> one arrival on the barrier at
// this offset in both CTAs of the pair.
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"((uint16_t)0x3)
      : "memory");
}
__device__ __forceinline__ void mma_commit_pair_local(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
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

// D (TMEM) += A (TMEM) * B (shared memory descriptor); PAIR = 2 issues the
// two-SM form (M = 256: A and D halves in each CTA's TMEM, B halves in each
// CTA's shared memory at the same offset).
template <int PAIR>
__device__ __forceinline__ void mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  if (PAIR == 1)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
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
template <class SM>
__device__ __forceinline__ TileId tile_id(const SM& sm, int E, int n_tiles, int t) {
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
template <class SM>
__device__ __forceinline__ TileInfo tile_info(const SM& sm, int E, int n_tiles, int t) {
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
// range where every scaled value is exact in fp16), INT4 the group's fp16
// scale (both halves; `bad` when not finite) and its zero as an fp16 pair.
template <int FMT>
__device__ __forceinline__ void stage_scales(uint32_t sc, uint32_t& h0, uint32_t& h1, uint32_t& zp,
                                             bool& bad) {
  if (FMT == kFmtNF4) {
    const float a = __uint_as_float(sc);
    bad |= a != 0.0f && !(a >= 6.103515625e-05f && a <= 65504.0f);
    const __half2 ah = __float2half2_rn(a);
    h0 = h1 = *reinterpret_cast<const uint32_t*>(&ah);
  } else if (FMT == kFmtMXFP4) {
    h0 = mx_scale_h2(sc & 0xFFu, bad);
    h1 = mx_scale_h2((sc >> 8) & 0xFFu, bad);
  } else {
    bad |= (sc & 0x7C00u) == 0x7C00u;
    h0 = h1 = (sc & 0xFFFFu) * 0x00010001u;
    const __half z = __uint2half_rn((sc >> 16) & 15u);
    zp = (uint32_t)(*reinterpret_cast<const uint16_t*>(&z)) * 0x00010001u;
  }
}

// TR = false: out[p, n] = sum_k W[e(p)][n, k] A[p, k] (the forward grouped
// GEMM; tiles of output rows n = weight rows).  TR = true: the transposed
// GEMM of the backward, out[p, k] = sum_n W[e(p)][n, k] A[p, n] (tiles of
// output columns k; A = the upstream gradient), NF4 only, single CTA; with
// EPI_SWIGLU_BWD its epilogue applies the SwiGLU backward to the result (the
// gradient of h) and writes the gradient of gate_up's pre-activations.
template <int FMT, int EPI, typename OutT, int PAIR, bool TR>
__global__ void __launch_bounds__(THREADS, 1) nf4_tc_kernel(
    const __grid_constant__ BMaps bmaps,
    const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap amap,
    const void* __restrict__ scales, const int32_t* __restrict__ offsets, int E, int N, int K,
    int M_total, OutT* __restrict__ out, const float* __restrict__ gu, int32_t* dev_err,
    int chain) {
  extern __shared__ uint8_t smem_raw[];
  if (!chain) {  // nothing is read or written before the previous kernel is done
    pdl_wait();
    pdl_trigger();
  }
  using Smem = SmemFor<OutT, TR>;
  constexpr int BSTAGES = Smem::kNBS;
  Smem& sm = *reinterpret_cast<Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // tiles of BM * PAIR output rows (weight rows; transposed: weight
  // columns); this CTA's 128-row part of tile ntile is sub-tile
  // ntile * PAIR + rank.  KT stages of BK along the reduction.
  const int n_tiles = (TR ? K : N) / (BM * PAIR);
  const int KT = (TR ? N : K) / BK;
  const int rank = PAIR == 1 ? 0 : (int)cluster_rank();
  const bool leader = rank == 0;
  const int t0 = blockIdx.x / PAIR, tstep = gridDim.x / PAIR;  // this pair's tiles

  // MMA N for a tile's routed rows: a multiple of 16 (one CTA) or of 32 (the
  // pair's M = 256 form, each CTA holding N / 2 rows of B)
  auto mma_n = [](int rows) { return PAIR == 1 ? (rows + 15) & ~15 : (rows + 31) & ~31; };

  // ---- setup: barriers, offsets, decode table, tile list, TMEM
  if (threadIdx.x == 0) {
    for (int s = 0; s < RAW_RING; ++s) {
      mbar_init(&sm.raw_full[s], 1);
      mbar_init(&sm.raw_empty[s], 4);   // the four warps of the decoding group
    }
    for (int s = 0; s < RING; ++s) {
      // the decoder warps of every CTA of the pair + the (leader's) B producer
      mbar_init(&sm.ready[s], 4 * PAIR + 1);
      mbar_init(&sm.a_empty[s], 1);     // MMA completion (tcgen05.commit)
    }
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.acc_empty, 32 * EPI_WARPS * PAIR);
    mbar_init(&sm.drain, 1);
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
    } else if (FMT == kFmtMXFP4) {
      sm.lut[i] = e2m1_h((uint32_t)b & 15u) | (e2m1_h((uint32_t)b >> 4) << 16);
    } else {  // INT4: the codes as exact fp16 integers {q(high nibble), q(low)}
      const __half2 h = __halves2half2(__uint2half_rn((unsigned)(b >> 4)),
                                       __uint2half_rn((unsigned)(b & 15)));
      sm.lut[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
  }
  if (warp == W_MMA) {
    if (PAIR == 1) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(&sm.tmem_base)),
                   "r"(TMEM_COLS));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    } else {  // same warp, same destination in both CTAs of the pair
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(&sm.tmem_base)),
                   "r"(TMEM_COLS));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
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
  if (PAIR == 2) cluster_sync();  // both CTAs' barriers and TMEM exist
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
      // Activation slot S mod BSTAGES is free once the MMAs of stage
      // S - BSTAGES are done: the a_empty barrier of that stage's TMEM slot
      // (one commit per stage serves both rings).  A stage is the rows the
      // tile's MMAs read (its routed rows rounded up to the MMA's N, a
      // multiple of 16; rows past the tile are loaded and never used), in
      // one box of exactly that height.  Pair form: each CTA loads its half
      // of them into its own slot; both halves are counted on the leader's
      // ready barrier.
      int bs = 0, S = 0;
      bool ok = true;
      for (int t = t0; t < total && ok; t += tstep) {
        const TileInfo ti = tile_info(sm, E, n_tiles, t);
        const int rows_b = mma_n(ti.nrows) / PAIR;  // 16 .. 256, a multiple of 16
        const CUtensorMap* bm = &bmaps.m[rows_b / 16 - 1];
        const int brow0 = ti.row0 + rank * rows_b;
        for (int ks = 0; ks < KT; ++ks, ++S) {
          if (S >= BSTAGES) {
            const int P = S - BSTAGES;
            // this thread paces the ring: it polls (single CTA) rather than
            // sleep in the barrier unit
            const uint32_t par = (uint32_t)(P / RING) & 1u;
            if (!(ok = PAIR == 1 ? mbar_poll(&sm.a_empty[P % RING], par, sm, dev_err)
                                 : mbar_wait<true>(&sm.a_empty[P % RING], par, sm, dev_err)))
              break;
          }
          uint64_t* rdy = &sm.ready[S % RING];
          // leader: its own barrier; the pair's peer: the leader's
          const uint32_t bar = leader ? smem_u32(rdy) : cluster_addr(rdy, 0);
          if (leader) mbar_arrive_expect_tx(rdy, PAIR * rows_b * BK * 2);
          if (PAIR == 1)
            tma_load_2d(sm.b[bs], bm, rdy, ks * BK, brow0);
          else
            tma_load_2d_pair(sm.b[bs], bm, bar, ks * BK, brow0);
          if (++bs == BSTAGES) bs = 0;
        }
      }
    }
  } else if (warp == W_MMA) {
    // ---------------- MMA issuer (the leader CTA's, in the pair form)
    if (lane == 0 && leader) {
      const uint64_t bdesc0 = sw128_desc(smem_u32(sm.b[0]));
      int bs = 0, as = 0;  // activation slot (as the producer's), TMEM slot
      uint32_t aph = 0;
      bool ok = true;
      int lt = 0;
      for (int t = t0; t < total && ok; t += tstep, ++lt) {
        const TileInfo ti = tile_info(sm, E, n_tiles, t);
        const int nmma = mma_n(ti.nrows);
        // the single accumulator must have been drained by the epilogue(s)
        if (!(ok = mbar_poll(&sm.acc_empty, (lt & 1) ^ 1, sm, dev_err))) break;
        tc_fence_after();
        const uint32_t idesc = idesc_f16(BM * PAIR, nmma);
        const uint32_t dcol = tmem_base + ACC_COL;
        for (int ks = 0; ks < KT; ++ks) {
          if (!(ok = mbar_poll(&sm.ready[as], aph, sm, dev_err))) break;
          tc_fence_after();
          // K slice kk: 8 more TMEM columns of A; 32 bytes further into the
          // swizzled activation rows (+2 in the descriptor's address field)
          const uint32_t acol = tmem_base + A_COL + as * A_SLOT_COLS;
          const uint64_t bd = bdesc0 + (uint64_t)((bs * B_STAGE) >> 4);
          mma_ts<PAIR>(dcol, acol, bd, idesc, ks != 0);
          mma_ts<PAIR>(dcol, acol + 8, bd + 2, idesc, 1u);
          mma_ts<PAIR>(dcol, acol + 16, bd + 4, idesc, 1u);
          mma_ts<PAIR>(dcol, acol + 24, bd + 6, idesc, 1u);
          // frees TMEM slot as and the stage's activation bytes (in both CTAs)
          if (PAIR == 1) mma_commit(&sm.a_empty[as]); else mma_commit_pair(&sm.a_empty[as]);
          if (++bs == BSTAGES) bs = 0;
          if (++as == RING) { as = 0; aph ^= 1; }
        }
        if (ok) {
          if (PAIR == 1) mma_commit(&sm.acc_full); else mma_commit_pair(&sm.acc_full);
        }
      }
      if (PAIR == 2) {
        // every MMA this thread issued has finished reading both CTAs'
        // shared and tensor memory before either CTA leaves
        // (bounded, and not cut short by an abort of another role)
        mma_commit_pair_local(&sm.drain);
        for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait_suspend_cl(&sm.drain, 0); ++i) {
        }
      }
    }
  } else if (warp == W_RPROD) {
    // ---------------- TMA producer: packed NF4 rows of the tile
    if (lane == 0) {
      // tile t's 128-row weight sub-tile of this CTA (wt) and the box
      // coordinates of its rows: forward SwiGLU y1 = z of the expert's gate
      // half; forward plain y0 = the first of 128 consecutive rows;
      // transposed y0 = the expert's first row
      auto tile_rows = [&](int t, int& wt, int& y0, int& y1) {
        const TileId id = tile_id(sm, E, n_tiles, t);
        wt = id.ntile * PAIR + rank;
        if (TR) {
          y0 = y1 = id.expert * N;
        } else if (EPI == MOE_EPI_SWIGLU) {
          y0 = 0;
          y1 = 2 * id.expert;  // z of the expert's gate half
        } else {
          y0 = id.expert * N + wt * BM;
          y1 = 0;
        }
      };
      int rs = 0;
      uint32_t rph = 0;
      bool ok = true;
      for (int t = t0; t < total && ok; t += tstep) {
        int wt, y0, y1;
        tile_rows(t, wt, y0, y1);
        for (int ks = 0; ks < KT; ++ks) {
          if (!(ok = mbar_wait(&sm.raw_empty[rs], rph ^ 1, sm, dev_err))) break;
          if (TR) {
            // weight rows n = 64 ks .. 64 ks + 63 of the expert, the packed
            // bytes of columns 128 wt .. 128 wt + 127, and the absmax of their
            // two 64-blocks (4 per row from a 16-byte-aligned block index)
            const int yr = y0 + ks * BK;
            mbar_arrive_expect_tx(&sm.raw_full[rs], RAW_STAGE_T);
            tma_load_2d(sm.raw[rs], &wmap, &sm.raw_full[rs], wt * (BM / 2), yr);
            tma_load_2d(sm.raw[rs] + RAW_STAGE, &amap, &sm.raw_full[rs], (2 * wt) & ~3, yr);
          } else if (EPI == MOE_EPI_SWIGLU) {
            // one 3-D box: the 64 gate rows, then the 64 matching up rows
            // (weight rows as [2E][N/2][K/2]: z = 2 expert + half)
            mbar_arrive_expect_tx(&sm.raw_full[rs], RAW_STAGE);
            tma_load_3d(sm.raw[rs], &wmap, &sm.raw_full[rs], ks * (BK / 2), wt * (BM / 2), y1);
          } else {
            // one box of the tile's 128 consecutive rows
            mbar_arrive_expect_tx(&sm.raw_full[rs], RAW_STAGE);
            tma_load_2d(sm.raw[rs], &wmap, &sm.raw_full[rs], ks * (BK / 2), y0);
          }
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
    if constexpr (TR) {
      // Transposed form: this thread's TMEM lane is output column
      // k = 128 wt + m; a stage's 32 columns of fp16 pairs are its weights in
      // rows n = 64 ks + 2c, 2c + 1, decoded from the byte of column k in each
      // row (high nibble for even k) through the byte table, times each row's
      // absmax of k's 64-block (fp16 products, as in the forward form).
      const uint32_t* lutl = sm.lut + lane;
      const int byte = m >> 1;
      // a table entry is {L[high nibble] (low half), L[low nibble] (high
      // half)}; even k takes the low halves of rows n and n + 1, odd k the
      // high halves
      const uint32_t sel = (m & 1) ? 0x7632u : 0x5410u;
      bool bad_scale = false;
      for (int S = g; ; S += GROUPS) {
        const int lt_ = S / KT;
        const int t = t0 + lt_ * tstep;
        if (t >= total) break;
        const TileId id = tile_id(sm, E, n_tiles, t);
        const int si = ((2 * id.ntile) & 3) + (m >> 6);  // absmax word of k's block
        const int slot = S % RING, rslot = S % RAW_RING;
        const uint32_t ph = (uint32_t)(S / RING) & 1u, rph = (uint32_t)(S / RAW_RING) & 1u;
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.raw_full[rslot], rph, sm, dev_err))) break;
        const uint8_t* rp = sm.raw[rslot];
        const float* sc = reinterpret_cast<const float*>(rp + RAW_STAGE);
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.a_empty[slot], ph ^ 1, sm, dev_err))) break;
        tc_fence_after();
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t hv[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int n = 32 * half + 2 * c;
            const uint32_t p0 = lutl[(uint32_t)rp[n * 64 + byte] << 5];
            const uint32_t p1 = lutl[(uint32_t)rp[(n + 1) * 64 + byte] << 5];
            const float a0 = sc[n * 4 + si], a1 = sc[(n + 1) * 4 + si];
            bad_scale |= (a0 != 0.0f && !(a0 >= 6.103515625e-05f && a0 <= 65504.0f)) ||
                         (a1 != 0.0f && !(a1 >= 6.103515625e-05f && a1 <= 65504.0f));
            const uint32_t lv = __byte_perm(p0, p1, sel);  // {L(row n), L(row n + 1)}
            const __half2 ah = __floats2half2_rn(a0, a1);
            const __half2 v = __hmul2(*reinterpret_cast<const __half2*>(&lv), ah);
            hv[c] = *reinterpret_cast<const uint32_t*>(&v);
          }
          tmem_st16(tlane + A_COL + slot * A_SLOT_COLS + 16 * half, hv);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sm.ready[slot]);
          mbar_arrive(&sm.raw_empty[rslot]);
        }
      }
      if (__any_sync(0xffffffffu, bad_scale) && lane == 0) set_dev_err(dev_err, MOE_DEVERR_RANGE);
    } else {
    // scales of this thread's weight row in tile t (null past the CTA's last
    // tile), stage ks at word ks: NF4 the fp32 absmax of block ks, MXFP4 the
    // two E8M0 bytes of the stage; walked one own stage ahead without
    // divisions
    auto row_scales = [&](int t) -> const uint8_t* {
      if (t >= total) return nullptr;
      const TileId id = tile_id(sm, E, n_tiles, t);
      const int wt = id.ntile * PAIR + rank;
      int row;
      if (EPI == MOE_EPI_SWIGLU) {
        const int j = wt * (BM / 2) + (m >> 1);
        row = (m & 1) ? (N / 2 + j) : j;
      } else {
        row = wt * BM + m;
      }
      const size_t r = (size_t)id.expert * N + row;
      return reinterpret_cast<const uint8_t*>(scales) +
             (FMT == kFmtNF4 ? r * (size_t)KT * 4
              : FMT == kFmtMXFP4 ? r * (size_t)(K / 32) : r * (size_t)(K / 128) * 4);
    };
    auto fetch = [&](const uint8_t* row, int ks) -> uint32_t {
      if (FMT == kFmtNF4) return __ldg(reinterpret_cast<const uint32_t*>(row) + ks);
      if (FMT == kFmtMXFP4) return __ldg(reinterpret_cast<const uint16_t*>(row) + ks);
      return __ldg(reinterpret_cast<const uint32_t*>(row) + (ks >> 1));  // 128-k group
    };
    int n_ks = g, n_t = t0;
    while (n_ks >= KT) { n_ks -= KT; n_t += tstep; }
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
        n_t += tstep;
        n_row = row_scales(n_t);
      }
      const bool have_next = n_row != nullptr;
      const uint32_t sc_next = have_next ? fetch(n_row, n_ks) : 0u;  // one stage ahead
      // warp-uniform outcomes: tcgen05.st below is .aligned
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.raw_full[rslot], rph, sm, dev_err))) break;
      const uint8_t* rp = sm.raw[rslot] + rrow * (BK / 2);
      const uint4 w0 = lds128(rp), w1 = lds128(rp + 16);
      uint32_t sh[2], zp = 0;
      stage_scales<FMT>(sc_cur, sh[0], sh[1], zp, bad_scale);
      if (!__all_sync(0xffffffffu, mbar_wait<PAIR == 2>(&sm.a_empty[slot], ph ^ 1, sm, dev_err)))
        break;
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
            __half2 lv = *reinterpret_cast<const __half2*>(&raw);
            if (FMT == kFmtINT4) lv = __hsub2(lv, *reinterpret_cast<const __half2*>(&zp));
            __half2 v = __hmul2(lv, ah);
            hv[4 * c + b] = *reinterpret_cast<uint32_t*>(&v);
          }
        }
        tmem_st16(tlane + A_COL + slot * A_SLOT_COLS + 16 * half, hv);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        // the slot is ready on the MMA-issuing CTA's barrier
        if (leader) mbar_arrive(&sm.ready[slot]);
        else mbar_arrive_remote(cluster_addr(&sm.ready[slot], 0));
        mbar_arrive(&sm.raw_empty[rslot]);  // its bytes are decoded
      }
      sc_cur = sc_next;
      have = have_next;
    }
    // the loop exits are warp-uniform, so every lane takes part
    if (__any_sync(0xffffffffu, bad_scale) && lane == 0) set_dev_err(dev_err, MOE_DEVERR_RANGE);
    }
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
    // the accumulator goes back to the MMA-issuing CTA
    auto release_acc = [&]() {
      tc_fence_before();
      if (leader) mbar_arrive(&sm.acc_empty);
      else mbar_arrive_remote(cluster_addr(&sm.acc_empty, 0));
    };
    for (int t = t0; t < total && ok; t += tstep, ++lt) {
      const TileInfo ti = tile_info(sm, E, n_tiles, t);
      if (!(ok = __all_sync(0xffffffffu,
                            mbar_wait<PAIR == 2>(&sm.acc_full, lt & 1, sm, dev_err))))
        break;
      tc_fence_after();
      const int ncols = mma_n(ti.nrows);
      // first output column of this warp's rows
      const int wt = ti.ntile * PAIR + rank;
      const int col0 = (EPI == MOE_EPI_SWIGLU) ? wt * (BM / 2) + 16 * q : wt * BM + 32 * q;
      // row pitch of out: SwiGLU N/2; transposed K, or 2K with the SwiGLU
      // backward (gate gradients at col, up gradients at K + col)
      const int ldo = (EPI == MOE_EPI_SWIGLU) ? N / 2
                      : TR ? (EPI == EPI_SWIGLU_BWD ? 2 * K : K) : N;
      // staged rows -> global, 16 bytes per lane, at column offset cofs
      auto store_staged = [&](int c0, int cofs) {
        __syncwarp();
#pragma unroll
        for (int idx = lane; idx < 32 * V; idx += 32) {
          const int tok = idx / V, piece = idx - tok * V;
          if (c0 + tok < ti.nrows) {
            const uint4 val = lds128(stg + tok * ROWB + piece * 16);
            *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(
                out + (size_t)(ti.row0 + c0 + tok) * ldo + cofs) + piece * 16) = val;
          }
        }
        __syncwarp();
      };
      bool released = false;
      for (int c0 = 32 * hc; c0 < ncols; c0 += 64) {
        uint32_t v[32];
        tmem_ld32(tmem_base + lane_addr + ACC_COL + c0, v);
        if (c0 + 64 >= ncols) {
          // this warp's last read of the accumulator: hand it back to the
          // MMA before the math and the stores
          release_acc();
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
        } else if (EPI == EPI_SWIGLU_BWD) {
          // v[i] = dh of token c0 + i at column col0 + lane; with s =
          // sigmoid(g): d gate = dh u s (1 + g (1 - s)), d up = dh g s, from
          // the forward's pre-activations gu [M, 2K] (fp32)
          float du[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const bool live = c0 + i < ti.nrows;
            const size_t gp = (size_t)(ti.row0 + c0 + i) * (2 * (size_t)K) + col0 + lane;
            const float gv = live ? __ldg(gu + gp) : 0.0f;
            const float uv = live ? __ldg(gu + gp + K) : 0.0f;
            const float sg = __fdiv_rn(1.0f, 1.0f + expf(-gv));
            const float dh = __uint_as_float(v[i]);
            const float dgate = dh * uv * sg * (1.0f + gv * (1.0f - sg));
            du[i] = dh * gv * sg;
            ovf |= live && (overflows_out<OutT>(dgate) || overflows_out<OutT>(du[i]));
            reinterpret_cast<OutT*>(stg + i * ROWB)[lane] = from_f32<OutT>(dgate);
          }
          store_staged(c0, col0);
#pragma unroll
          for (int i = 0; i < 32; ++i)
            reinterpret_cast<OutT*>(stg + i * ROWB)[lane] = from_f32<OutT>(du[i]);
          store_staged(c0, K + col0);
          continue;
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float y = __uint_as_float(v[i]);
            ovf |= c0 + i < ti.nrows && overflows_out<OutT>(y);
            reinterpret_cast<OutT*>(stg + i * ROWB)[lane] = from_f32<OutT>(y);
          }
        }
        store_staged(c0, col0);
      }
      if (!released) release_acc();  // no columns for this warp in this tile
    }
    // the loop exits are warp-uniform, so every lane takes part
    if (__any_sync(0xffffffffu, ovf) && lane == 0) set_dev_err(dev_err, MOE_DEVERR_RANGE);
  }

  // single-lane roles (producers, MMA issuer) rejoin their warp before the
  // CTA-wide barrier; in the pair form neither CTA frees its tensor memory or
  // leaves (its shared memory holds barriers the other CTA arrives on) before
  // both are done
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (PAIR == 2) cluster_sync();
  if (warp == W_MMA) {
    tc_fence_after();
    if (PAIR == 1)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"(TMEM_COLS));
    else
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"(TMEM_COLS));
  }
}

int sm_count() { return device_sm_count(); }

// Clusters of two of `kern` that fit on the device at once, once per kernel
// and device (the GPCs' SM counts decide it); SMs / 2 if the query fails.
inline int max_pair_clusters(const void* kern, size_t smem) {
  static std::mutex mu;
  static std::unordered_map<uint64_t, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return std::max(1, sm_count() / 2);
  const uint64_t key = (reinterpret_cast<uint64_t>(kern) << 6) ^ (uint64_t)dev;
  {
    std::lock_guard<std::mutex> lock(mu);
    const auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * std::max(1, sm_count() / 2));
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
    (void)cudaGetLastError();
    n = std::max(1, sm_count() / 2);
  }
  std::lock_guard<std::mutex> lock(mu);
  cache[key] = n;
  return n;
}

template <int FMT, int EPI, typename OutT, int PAIR>
cudaError_t launch(const void* A, const uint8_t* packed, const void* scales,
                   const int32_t* offsets, int E, int N, int K, int M_total, void* out,
                   int32_t* dev_err, cudaStream_t s, bool chain) {
  if (!tensor_map_encoder()) return cudaErrorNotSupported;
  const auto enc = encode_tiled_cached;
  BMaps bmaps;
  CUtensorMap wmap;
  const cuuint32_t estr[3] = {1, 1, 1};
  for (int i = 0; i < B_MAPS; ++i) {
    // routed activation rows: boxes of 64 k x 16 (i + 1) rows
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M_total};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {BK, (cuuint32_t)(16 * (i + 1))};
    if (enc(&bmaps.m[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
            const_cast<void*>(A), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  if (EPI == MOE_EPI_SWIGLU) {
    // packed rows as [2E][N/2][K/2] (z = 2 expert + half); box = 32 bytes x
    // 64 rows x 2 halves: a stage's gate rows and their up rows in one copy
    const cuuint64_t dims[3] = {(cuuint64_t)K / 2, (cuuint64_t)N / 2, (cuuint64_t)2 * E};
    const cuuint64_t strides[2] = {(cuuint64_t)K / 2, (cuuint64_t)(N / 2) * (K / 2)};
    const cuuint32_t box[3] = {BK / 2, BM / 2, 2};
    if (enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(packed), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    // packed rows as a 2-D byte tensor [E*N, K/2]; box = 32 bytes x 128 rows
    const cuuint64_t dims[2] = {(cuuint64_t)K / 2, (cuuint64_t)E * N};
    const cuuint64_t strides[1] = {(cuuint64_t)K / 2};
    const cuuint32_t box[2] = {BK / 2, BM};
    if (enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(packed), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const size_t smem = sizeof(SmemFor<OutT, false>) + 1024;
  auto kern = nf4_tc_kernel<FMT, EPI, OutT, PAIR, false>;
  cudaError_t err = set_max_dynamic_smem_once(reinterpret_cast<const void*>(kern), (int)smem);
  if (err != cudaSuccess) return err;
  // Upper bound on tiles: every expert's rows rounded up to BN, plus one
  // partial tile per expert; the kernel derives the exact list itself.
  const int64_t max_tiles = ((int64_t)M_total / BN + E) * (N / (BM * PAIR));
  if (PAIR == 1) {
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(sm_count(), max_tiles));
    return launch_pdl(kern, dim3(grid), dim3(THREADS), smem, s, bmaps, wmap, wmap, scales,
                      offsets, E, N, K, M_total, reinterpret_cast<OutT*>(out),
                      static_cast<const float*>(nullptr), dev_err, chain ? 1 : 0);
  }
  const int clusters = (int)std::max<int64_t>(
      1, std::min<int64_t>(max_pair_clusters(reinterpret_cast<const void*>(kern), smem),
                           max_tiles));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, bmaps, wmap, wmap, scales, offsets, E, N, K, M_total,
                            reinterpret_cast<OutT*>(out), static_cast<const float*>(nullptr),
                            dev_err, chain ? 1 : 0);
}

// The transposed (backward) form: out[p, k] = sum_n W[e(p)][n, k] G[p, n],
// G fp16 [G_rows, N] in permuted order; EPI_SWIGLU_BWD applies the SwiGLU
// backward with gu fp32 [M_total, 2K] and writes out [M_total, 2K].
template <int EPI, typename OutT>
cudaError_t launch_t(const void* G, int G_rows, const uint8_t* packed, const float* absmax,
                     const int32_t* offsets, int E, int N, int K, int M_total, void* out,
                     const float* gu, int32_t* dev_err, cudaStream_t s) {
  if (!tensor_map_encoder()) return cudaErrorNotSupported;
  const auto enc = encode_tiled_cached;
  BMaps bmaps;
  CUtensorMap wmap, amap;
  const cuuint32_t estr[2] = {1, 1};
  for (int i = 0; i < B_MAPS; ++i) {
    const cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)G_rows};
    const cuuint64_t strides[1] = {(cuuint64_t)N * 2};
    const cuuint32_t box[2] = {BK, (cuuint32_t)(16 * (i + 1))};
    if (enc(&bmaps.m[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
            const_cast<void*>(G), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    // packed rows [E*N, K/2]; box = 64 bytes (128 columns) x 64 rows
    const cuuint64_t dims[2] = {(cuuint64_t)K / 2, (cuuint64_t)E * N};
    const cuuint64_t strides[1] = {(cuuint64_t)K / 2};
    const cuuint32_t box[2] = {BM / 2, BK};
    if (enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(packed), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    // absmax [E*N, K/64]; box = 4 blocks x 64 rows
    const cuuint64_t dims[2] = {(cuuint64_t)K / kBlock, (cuuint64_t)E * N};
    const cuuint64_t strides[1] = {(cuuint64_t)K / kBlock * 4};
    const cuuint32_t box[2] = {4, BK};
    if (enc(&amap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(absmax), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const size_t smem = sizeof(SmemFor<OutT, true>) + 1024;
  auto kern = nf4_tc_kernel<kFmtNF4, EPI, OutT, 1, true>;
  cudaError_t err = set_max_dynamic_smem_once(reinterpret_cast<const void*>(kern), (int)smem);
  if (err != cudaSuccess) return err;
  const int64_t max_tiles = ((int64_t)M_total / BN + E) * (K / BM);
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(sm_count(), max_tiles));
  return launch_pdl(kern, dim3(grid), dim3(THREADS), smem, s, bmaps, wmap, amap,
                    static_cast<const void*>(absmax), offsets, E, N, K, M_total,
                    reinterpret_cast<OutT*>(out), gu, dev_err, 0);
}

template <int FMT, int EPI, typename OutT>
cudaError_t launch_pair_or_not(const void* A, const uint8_t* packed, const void* scales,
                               const int32_t* offsets, int E, int N, int K, int M_total,
                               void* out, int32_t* dev_err, cudaStream_t s, bool chain,
                               bool pair) {
  // the pair form needs whole 256-row weight tiles
  if (pair && N % (2 * BM) == 0)
    return launch<FMT, EPI, OutT, 2>(A, packed, scales, offsets, E, N, K, M_total, out, dev_err,
                                     s, chain);
  return launch<FMT, EPI, OutT, 1>(A, packed, scales, offsets, E, N, K, M_total, out, dev_err, s,
                                   chain);
}

template <int FMT>
cudaError_t launch_fmt(const void* A, const uint8_t* packed, const void* scales,
                       const int32_t* offsets, int E, int N, int K, int M_total,
                       moe_epilogue_t epi, void* out, moe_dtype_t out_dt, int32_t* dev_err,
                       cudaStream_t s, bool chain, bool pair) {
  if (epi == MOE_EPI_SWIGLU) {
    if (out_dt == MOE_DT_F16)
      return launch_pair_or_not<FMT, MOE_EPI_SWIGLU, __half>(A, packed, scales, offsets, E, N, K,
                                                             M_total, out, dev_err, s, chain, pair);
    if (out_dt == MOE_DT_BF16)
      return launch_pair_or_not<FMT, MOE_EPI_SWIGLU, __nv_bfloat16>(
          A, packed, scales, offsets, E, N, K, M_total, out, dev_err, s, chain, pair);
    return launch_pair_or_not<FMT, MOE_EPI_SWIGLU, float>(A, packed, scales, offsets, E, N, K,
                                                          M_total, out, dev_err, s, chain, pair);
  }
  if (out_dt == MOE_DT_F16)
    return launch_pair_or_not<FMT, MOE_EPI_NONE, __half>(A, packed, scales, offsets, E, N, K,
                                                         M_total, out, dev_err, s, chain, pair);
  if (out_dt == MOE_DT_BF16)
    return launch_pair_or_not<FMT, MOE_EPI_NONE, __nv_bfloat16>(A, packed, scales, offsets, E, N,
                                                                K, M_total, out, dev_err, s,
                                                                chain, pair);
  return launch_pair_or_not<FMT, MOE_EPI_NONE, float>(A, packed, scales, offsets, E, N, K,
                                                      M_total, out, dev_err, s, chain, pair);
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
                            cudaStream_t s, bool chain, bool pair) {
  (void)k;
  if (gather || a_dt != MOE_DT_F16 || A_rows < M_total) return cudaErrorNotSupported;
  return moe::tc::launch_fmt<moe::kFmtNF4>(A, packed, absmax, offsets, E, N, K, M_total, epi,
                                           out, out_dt, dev_err, s, chain, pair);
}

bool grouped_gemm_t_tc_supported(int N, int K) {
  // 128-column output tiles, 64-row reduction stages, and an absmax row
  // pitch that is a multiple of 16 bytes (the TMA stride rule)
  return N % moe::tc::BK == 0 && N >= moe::tc::BK && K % 256 == 0;
}

cudaError_t grouped_gemm_t_tc(const void* G, int G_rows, const uint8_t* packed,
                              const float* absmax, const int32_t* offsets, int E, int N, int K,
                              int M_total, bool swiglu_bwd, const float* gu, void* out,
                              moe_dtype_t out_dt, int32_t* dev_err, cudaStream_t s) {
  using namespace moe::tc;
  if (G_rows < M_total) return cudaErrorNotSupported;
  if (swiglu_bwd) {
    if (out_dt == MOE_DT_F16)
      return launch_t<EPI_SWIGLU_BWD, __half>(G, G_rows, packed, absmax, offsets, E, N, K,
                                              M_total, out, gu, dev_err, s);
    return launch_t<EPI_SWIGLU_BWD, float>(G, G_rows, packed, absmax, offsets, E, N, K, M_total,
                                           out, gu, dev_err, s);
  }
  if (out_dt == MOE_DT_F16)
    return launch_t<MOE_EPI_NONE, __half>(G, G_rows, packed, absmax, offsets, E, N, K, M_total,
                                          out, nullptr, dev_err, s);
  return launch_t<MOE_EPI_NONE, float>(G, G_rows, packed, absmax, offsets, E, N, K, M_total, out,
                                       nullptr, dev_err, s);
}

cudaError_t grouped_gemm_tc_int4(const void* A, int A_rows, const uint8_t* packed,
                                 const uint32_t* meta, const int32_t* offsets, int E, int N,
                                 int K, int M_total, moe_epilogue_t epi, void* out,
                                 moe_dtype_t out_dt, int32_t* dev_err, cudaStream_t s) {
  if (A_rows < M_total) return cudaErrorNotSupported;
  return moe::tc::launch_fmt<moe::kFmtINT4>(A, packed, meta, offsets, E, N, K, M_total, epi, out,
                                            out_dt, dev_err, s, false, false);
}

cudaError_t grouped_gemm_tc_mxfp4(const void* A, int A_rows, const uint8_t* packed,
                                  const uint8_t* scales, const int32_t* offsets, int E, int N,
                                  int K, int M_total, moe_epilogue_t epi, void* out,
                                  moe_dtype_t out_dt, int32_t* dev_err, cudaStream_t s,
                                  bool pair) {
  if (A_rows < M_total) return cudaErrorNotSupported;
  return moe::tc::launch_fmt<moe::kFmtMXFP4>(A, packed, scales, offsets, E, N, K, M_total, epi,
                                             out, out_dt, dev_err, s, false, pair);
}

}  // namespace moe_launch
