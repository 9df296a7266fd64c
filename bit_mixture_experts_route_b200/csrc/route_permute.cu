// Top-k softmax routing and the stable token->expert permutation.
//
// The router of "grouped-nf4-gemm & experts-4bit" (jordananderson-pages
// .pages.dev, second bullet) feeds a kernel that covers all active experts
// in one launch (first bullet); that launch reads each expert's routed rows
// as one contiguous segment, which this file builds:
//   expert_offsets[E+1]  segment starts (exclusive scan of per-expert counts)
//   sorted_rows[T*k]     flat ids t*k+j ordered by expert, then by flat id
//   inv_perm[T*k]        position of each flat id
//
// Decode sizes (T*k <= 4096, E <= 256) run in one single-CTA launch
// (route_small_kernel).  Larger problems take two launches, both
// deterministic (no atomics whose order matters):
//  1. route_tile_kernel, one CTA per tile of 64 tokens: one warp per token
//     selects the top-k with 64-bit keys (ordered logit, ~expert) so ties go
//     to the lower expert and every lane agrees even on NaN (two redux.sync
//     maxima per selection), computes the
//     softmax weights, then warp 0 ranks the tile's routed rows stably with
//     __match_any_sync and writes the tile's per-expert counts.
//  2. permute_scatter_kernel, one CTA per tile: sums the tile counts into
//     expert totals and the tile's prefix, scans the totals into offsets and
//     scatters each flat id to offsets[e] + prefix + rank.
#include <climits>
#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kTileTok = 64;  // tokens per routing tile / CTA
constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t ordered_bits(float v) {
  const uint32_t u = __float_as_uint(v + 0.0f);  // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float unordered_bits(uint32_t o) {
  const uint32_t u = (o & 0x80000000u) ? (o & 0x7fffffffu) : ~o;
  return __uint_as_float(u);
}

// Top-k of one token's logits by one warp.  Lane l holds experts l + 32 i
// as 64-bit keys (order-preserving logit bits << 32 | ~expert; 0 = absent),
// so the largest key is the largest logit and, among equal logits, the lower
// expert.  Each of the k rounds takes the warp maximum in two redux.sync
// steps (high word, then low word among the lanes holding that high word).
// Lane j < k receives the j-th selected key in `mine`; every lane receives
// the largest key in `first`.
template <int NPER>
__device__ __forceinline__ void warp_topk(const uint64_t (&key)[NPER], int k, int E,
                                          uint64_t& mine, uint64_t& first) {
  const int lane = threadIdx.x & 31;
  uint32_t taken = 0;
  mine = 0;
  first = 0;
  for (int j = 0; j < k; ++j) {
    uint64_t best = 0;
#pragma unroll
    for (int i = 0; i < NPER; ++i)
      if (!((taken >> i) & 1u) && key[i] > best) best = key[i];
    const uint32_t hi = (uint32_t)(best >> 32);
    const uint32_t mh = __reduce_max_sync(0xffffffffu, hi);
    const uint32_t ml = __reduce_max_sync(0xffffffffu, hi == mh ? (uint32_t)best : 0u);
    const uint64_t sel = ((uint64_t)mh << 32) | ml;
    const int e = (int)(~ml);
    if (e >= 0 && e < E && (e & 31) == lane) taken |= 1u << (e >> 5);
    if (j == lane) mine = sel;
    if (j == 0) first = sel;
  }
}

// Routing weights of the selected experts (softmax over the k selected
// logits when renormalising, else over all E); lane j < k returns weight j.
template <int NPER>
__device__ __forceinline__ float warp_topk_weight(const uint64_t (&key)[NPER], uint64_t mine,
                                                  uint64_t first, int k, int E, int renorm) {
  const int lane = threadIdx.x & 31;
  const float mx = unordered_bits((uint32_t)(first >> 32));
  float ex = 0.0f;
  if (lane < k) ex = expf(unordered_bits((uint32_t)(mine >> 32)) - mx);
  float denom;
  if (renorm) {
    denom = warp_sum(ex);
  } else {
    float part = 0.0f;
#pragma unroll
    for (int i = 0; i < NPER; ++i)
      if (lane + 32 * i < E) part += expf(unordered_bits((uint32_t)(key[i] >> 32)) - mx);
    denom = warp_sum(part);
  }
  return __fdiv_rn(ex, denom);
}

template <int NPER>
__device__ __forceinline__ void load_keys(const float* row, int E, uint64_t (&key)[NPER]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < NPER; ++i) {
    const int e = lane + 32 * i;
    key[i] = (e < E) ? ((uint64_t)ordered_bits(row[e]) << 32) | (uint32_t)(~e) : 0ull;
  }
}

template <int NPER>
__global__ void __launch_bounds__(kThreads) route_tile_kernel(
    const float* __restrict__ logits, int T, int E, int k, int renorm,
    int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
    int32_t* __restrict__ rank, int32_t* __restrict__ tile_counts) {
  pdl_wait();
  pdl_trigger();
  __shared__ int s_eid[kTileTok * 32];
  __shared__ int s_cnt[1024];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tile = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += kThreads) s_cnt[e] = 0;

  for (int tt = warp; tt < kTileTok; tt += kThreads / 32) {
    const int t = tile * kTileTok + tt;
    if (t >= T) break;
    uint64_t key[NPER];
    load_keys<NPER>(logits + (size_t)t * E, E, key);
    uint64_t mine, first;
    warp_topk<NPER>(key, k, E, mine, first);
    const float w = warp_topk_weight<NPER>(key, mine, first, k, E, renorm);
    if (lane < k) {
      const int e = (int)(~(uint32_t)mine);
      topk_idx[(size_t)t * k + lane] = e;
      topk_w[(size_t)t * k + lane] = w;
      s_eid[tt * k + lane] = e;
    }
  }
  __syncthreads();

  // Stable rank of every routed row of the tile within its expert: one warp
  // walks the tile in flat order, 32 rows at a time.
  const int ntok = min(kTileTok, T - tile * kTileTok);
  const int n = ntok * k;
  const size_t fbase = (size_t)tile * kTileTok * k;
  if (warp == 0) {
    for (int base = 0; base < n; base += 32) {
      const int f = base + lane;
      int e = (f < n) ? s_eid[f] : -1;
      const bool valid = (e >= 0 && e < E);
      const int keyv = valid ? e : (1 << 20) + lane;  // unique for invalid lanes
      const unsigned peers = __match_any_sync(0xffffffffu, keyv);
      const int r = __popc(peers & lanemask_lt());
      const int c0 = valid ? s_cnt[e] : 0;
      __syncwarp();
      if (valid && (peers >> lane) == 1u) s_cnt[e] = c0 + __popc(peers);  // last lane of group
      __syncwarp();
      if (f < n) rank[fbase + f] = valid ? c0 + r : -1;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kThreads) tile_counts[(size_t)tile * E + e] = s_cnt[e];
}

// Decode-sized routing in one launch (T*k <= kSmallRows, E <= kSmallE): one
// CTA of 32 warps routes every token (warp per token), ranks the routed rows
// stably (each warp walks a contiguous chunk of flat ids with
// __match_any_sync, keeping per-warp expert counts), scans the counts into
// expert offsets and scatters.
constexpr int kSmallRows = 4096;
constexpr int kSmallE = 256;
constexpr int kSmallThreads = 1024;

template <int NPER>
__global__ void __launch_bounds__(kSmallThreads) route_small_kernel(
    const float* __restrict__ logits, int T, int E, int k, int renorm,
    int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
    int32_t* __restrict__ offsets, int32_t* __restrict__ sorted_rows,
    int32_t* __restrict__ inv_perm) {
  pdl_wait();
  pdl_trigger();
  // 16-bit fields: rows, ranks and counts are all < kSmallRows = 4096
  __shared__ int16_t s_eid[kSmallRows];
  __shared__ uint16_t s_rank[kSmallRows];
  __shared__ uint16_t s_wc[32][kSmallE];   // per-warp expert counts, then prefixes
  __shared__ int s_off[kSmallE + 1];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < 32 * kSmallE; i += kSmallThreads) (&s_wc[0][0])[i] = 0;
  // (made visible by the __syncthreads after the routing loop)

  for (int t = warp; t < T; t += 32) {
    uint64_t key[NPER];
    load_keys<NPER>(logits + (size_t)t * E, E, key);
    uint64_t mine, first;
    warp_topk<NPER>(key, k, E, mine, first);
    const float w = warp_topk_weight<NPER>(key, mine, first, k, E, renorm);
    if (lane < k) {
      const int e = (int)(~(uint32_t)mine);
      topk_idx[(size_t)t * k + lane] = e;
      topk_w[(size_t)t * k + lane] = w;
      s_eid[t * k + lane] = (int16_t)((e >= 0 && e < E) ? e : -1);
    }
  }
  __syncthreads();

  // stable rank within each warp's contiguous chunk of flat ids
  const int n = T * k;
  const int chunk = (n + 31) / 32;
  const int f0 = warp * chunk, f1 = min(n, f0 + chunk);
  for (int base = f0; base < f1; base += 32) {
    const int f = base + lane;
    const int e = (f < f1) ? s_eid[f] : -1;
    const bool valid = e >= 0 && e < E;
    const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : (1 << 20) + lane);
    const int r = __popc(peers & lanemask_lt());
    const int c0 = valid ? s_wc[warp][e] : 0;
    __syncwarp();
    if (valid && (peers >> lane) == 1u) s_wc[warp][e] = (uint16_t)(c0 + __popc(peers));
    __syncwarp();
    if (f < f1) s_rank[f] = valid ? (uint16_t)(c0 + r) : (uint16_t)0xffffu;
  }
  __syncthreads();

  // per expert: exclusive prefix over warps, and the total
  if (threadIdx.x < E) {
    const int e = threadIdx.x;
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      const int c = s_wc[w][e];
      s_wc[w][e] = (uint16_t)run;
      run += c;
    }
    s_off[e] = run;
  }
  __syncthreads();
  // exclusive scan of the totals by warp 0 (E <= 256: 8 per lane)
  if (warp == 0) {
    int v[kSmallE / 32];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < kSmallE / 32; ++i) {
      const int e = lane * (kSmallE / 32) + i;
      v[i] = e < E ? s_off[e] : 0;
      sum += v[i];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - sum;
#pragma unroll
    for (int i = 0; i < kSmallE / 32; ++i) {
      const int e = lane * (kSmallE / 32) + i;
      if (e < E) s_off[e] = run;
      run += v[i];
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e <= E; e += kSmallThreads) offsets[e] = (e < E) ? s_off[e] : n;
  for (int f = threadIdx.x; f < n; f += kSmallThreads) {
    const int e = s_eid[f];
    const int r = s_rank[f];
    if (e < 0 || e >= E || r == 0xffff) continue;
    const int pos = s_off[e] + s_wc[f / chunk][e] + r;
    if (pos < 0 || pos >= n) continue;
    sorted_rows[pos] = f;
    inv_perm[f] = pos;
  }
}

// Exclusive scan of s[0..n) in place for n <= 1024 with kThreads threads.
__device__ void block_exclusive_scan(int* s, int n, int* s_warp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kPer = 1024 / kThreads;  // 4 elements per thread
  int v[kPer];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int idx = threadIdx.x * kPer + i;
    v[i] = idx < n ? s[idx] : 0;
    sum += v[i];
  }
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kThreads / 32 ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kThreads / 32) s_warp[lane] = w;  // inclusive warp totals
  }
  __syncthreads();
  int run = incl - sum + (warp ? s_warp[warp - 1] : 0);
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int idx = threadIdx.x * kPer + i;
    if (idx < n) s[idx] = run;
    run += v[i];
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kThreads) permute_scatter_kernel(
    const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ rank,
    const int32_t* __restrict__ tile_counts, int T, int E, int k, int ntiles,
    int32_t* __restrict__ offsets, int32_t* __restrict__ sorted_rows,
    int32_t* __restrict__ inv_perm) {
  pdl_wait();
  pdl_trigger();
  __shared__ int s_off[1024];
  __shared__ int s_before[1024];
  __shared__ int s_warp[kThreads / 32];
  const int tile = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += kThreads) {
    int tot = 0, before = 0;
    for (int b = 0; b < ntiles; ++b) {
      const int c = tile_counts[(size_t)b * E + e];
      before += (b < tile) ? c : 0;
      tot += c;
    }
    s_off[e] = tot;
    s_before[e] = before;
  }
  __syncthreads();
  block_exclusive_scan(s_off, E, s_warp);
  if (tile == 0) {
    for (int e = threadIdx.x; e < E; e += kThreads) offsets[e] = s_off[e];
    if (threadIdx.x == 0) offsets[E] = T * k;
  }
  for (int e = threadIdx.x; e < E; e += kThreads) s_before[e] += s_off[e];
  __syncthreads();
  const int ntok = min(kTileTok, T - tile * kTileTok);
  const int n = ntok * k;
  const size_t fbase = (size_t)tile * kTileTok * k;
  const int total = T * k;
  for (int i = threadIdx.x; i < n; i += kThreads) {
    const size_t f = fbase + i;
    const int e = topk_idx[f];
    const int r = rank[f];
    if (e < 0 || e >= E || r < 0) continue;
    const int pos = s_before[e] + r;
    if (pos < 0 || pos >= total) continue;
    sorted_rows[pos] = (int32_t)f;
    inv_perm[f] = pos;
  }
}

}  // namespace
}  // namespace moe

namespace moe_launch {

static size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

size_t route_workspace_bytes(int T, int E, int k) {
  const size_t ntiles = (T + moe::kTileTok - 1) / moe::kTileTok;
  return align256((size_t)T * k * 4) + align256(ntiles * E * 4);
}

cudaError_t route_permute(const float* logits, int T, int E, int k, int renorm,
                          int32_t* topk_idx, float* topk_w, int32_t* offsets,
                          int32_t* sorted_rows, int32_t* inv_perm, void* ws,
                          cudaStream_t s) {
  if (T == 0) return cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), s);
  if ((int64_t)T * k <= moe::kSmallRows && E <= moe::kSmallE) {
#define MOE_ROUTE_SMALL(NP)                                                             \
  moe::launch_pdl(moe::route_small_kernel<NP>, dim3(1), dim3(moe::kSmallThreads), 0, s, logits, \
                  T, E, k, renorm, topk_idx, topk_w, offsets, sorted_rows, inv_perm)
    if (E <= 32) return MOE_ROUTE_SMALL(1);
    if (E <= 64) return MOE_ROUTE_SMALL(2);
    if (E <= 128) return MOE_ROUTE_SMALL(4);
    return MOE_ROUTE_SMALL(8);
#undef MOE_ROUTE_SMALL
  }
  const int ntiles = (T + moe::kTileTok - 1) / moe::kTileTok;
  int32_t* rank = reinterpret_cast<int32_t*>(ws);
  int32_t* tile_counts =
      reinterpret_cast<int32_t*>(reinterpret_cast<char*>(ws) + align256((size_t)T * k * 4));
#define MOE_ROUTE_LAUNCH(NP)                                                           \
  moe::launch_pdl(moe::route_tile_kernel<NP>, dim3(ntiles), dim3(moe::kThreads), 0, s, logits, \
                  T, E, k, renorm, topk_idx, topk_w, rank, tile_counts)
  cudaError_t err;
  if (E <= 32) err = MOE_ROUTE_LAUNCH(1);
  else if (E <= 64) err = MOE_ROUTE_LAUNCH(2);
  else if (E <= 128) err = MOE_ROUTE_LAUNCH(4);
  else if (E <= 256) err = MOE_ROUTE_LAUNCH(8);
  else if (E <= 512) err = MOE_ROUTE_LAUNCH(16);
  else err = MOE_ROUTE_LAUNCH(32);
#undef MOE_ROUTE_LAUNCH
  if (err != cudaSuccess) return err;
  return moe::launch_pdl(moe::permute_scatter_kernel, dim3(ntiles), dim3(moe::kThreads), 0, s,
                         topk_idx, rank, tile_counts, T, E, k, ntiles, offsets, sorted_rows,
                         inv_perm);
}

// ---------------------------------------------------------------------------
// Routing without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they route:
// a host framework that owns every byte of device memory through its own
// allocator and forbids side allocations, or a latency-critical serving loop
// in which cudaMalloc (which may synchronize the device) is not acceptable.
// For them the routing scratch (per-row ranks and per-tile expert counts)
// lives in one fixed-size array in this library's device memory instead.
// Every GPU that loads the library holds this array until the process exits.
// ---------------------------------------------------------------------------

namespace {

__device__ __align__(256) unsigned char g_route_scratch[MOE_ROUTE_NOALLOC_SCRATCH_BYTES];

// The array's device address in each CUDA context, looked up once per
// context.  A __device__ variable has one address per context (normally a
// device's primary context, but a caller may make another context current),
// so the cache is keyed by the context that is current when the call runs.
// In host code `g_route_scratch` only names a host-side stand-in, so the
// kernel must be given the address that cudaGetSymbolAddress reports.
std::mutex g_scratch_mu;
constexpr int kMaxContexts = 64;
CUcontext g_scratch_ctx[kMaxContexts] = {};
void* g_scratch_addr[kMaxContexts] = {};
int g_scratch_n = 0;

// cuCtxGetCurrent from the driver, looked up once through the runtime (the
// library has no link-time dependency on libcuda).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  return fn;
}

cudaError_t scratch_for_current_context(void** out) {
  const CtxGetCurrentFn get_ctx = ctx_get_current();
  if (!get_ctx) return cudaErrorNotSupported;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return cudaErrorInitializationError;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (ctx) {
    for (int i = 0; i < g_scratch_n; ++i)
      if (g_scratch_ctx[i] == ctx) {
        *out = g_scratch_addr[i];
        return cudaSuccess;
      }
  }
  // First call in this context (or no context yet: the runtime then makes
  // the current device's primary context current while it looks the symbol
  // up).
  void* p = nullptr;
  cudaError_t err = cudaGetSymbolAddress(&p, g_route_scratch);
  if (err != cudaSuccess) return err;
  if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorInitializationError;
  if (g_scratch_n < kMaxContexts) {
    g_scratch_ctx[g_scratch_n] = ctx;
    g_scratch_addr[g_scratch_n] = p;
    ++g_scratch_n;
  }
  *out = p;
  return cudaSuccess;
}

}  // namespace

bool route_noalloc_fits(int T, int E, int k) {
  return route_workspace_bytes(T, E, k) <= (size_t)MOE_ROUTE_NOALLOC_SCRATCH_BYTES;
}

cudaError_t route_permute_noalloc(const float* logits, int T, int E, int k, int renorm,
                                  int32_t* topk_idx, float* topk_w, int32_t* offsets,
                                  int32_t* sorted_rows, int32_t* inv_perm, cudaStream_t s) {
  void* ws = nullptr;
  cudaError_t err = scratch_for_current_context(&ws);
  if (err != cudaSuccess) return err;
  // Nothing in the scratch has to start at zero: the routing kernel writes
  // every rank and every tile count before the scatter kernel reads them, so
  // contents left by an earlier call are never observed.
  return route_permute(logits, T, E, k, renorm, topk_idx, topk_w, offsets, sorted_rows,
                       inv_perm, ws, s);
}

}  // namespace moe_launch
