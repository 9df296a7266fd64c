// Per-expert LoRA delta over the routed rows (fp16 adapters, fp32 sums).
//
// The pages fine-tune the 4-bit mixture with a LoRA adapter per expert over
// the frozen base weights ("Jordan Anderson", jordananderson.work, section
// "4-bit Mixture-of-Experts fine-tuning on small GPUs"; "MoE Training on
// Consumer GPUs", cerinamroth.com/ml).  In LoRA's form the adapted projection
// of routed row p of expert e is W_e x_p + scale * B_e (A_e x_p).  The grouped
// GEMM writes the first term (fp32, no epilogue); this kernel adds the second
// to it in place, before SiLU(gate) * up.
//
// One CTA per (tile of up to R rows of one expert's segment, column split).
//   Phase 1: u[i][j] = scale * (A_e[j] . x_{p0+i}) for the tile's rows, fp32.  Each warp
//     takes a 4-row x 4-rank block at a time; lanes split K in 8-element
//     (16-byte) vectors and a warp reduction writes the block to shared memory.
//   Phase 2: each thread owns output columns n of the CTA's split and adds
//     sum_j B_e[n][j] u[i][j] to out[p0+i][n], accumulating onto the loaded value.
// The adapters are tiny next to the 4-bit base (r (N + K) fp16 values per
// expert against N K / 2 bytes); decode is bound by reading them and the fp32
// pre-activation, prefill by the r (N + K) multiply-adds per row.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kLoraThreads = 256;
constexpr int kLoraWarps = kLoraThreads / 32;
constexpr int kLoraMaxRank = 64;
constexpr int kLoraMaxE = 1024;

__device__ __forceinline__ void h8_to_f32(const uint4& v, float (&f)[8]) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 t = __half22float2(h[q]);
    f[2 * q] = t.x;
    f[2 * q + 1] = t.y;
  }
}

// fp32 FMA of four 8-element x vectors against four 8-element a vectors
__device__ __forceinline__ void dot4x4(const uint4 (&xr)[4], const uint4 (&ar)[4],
                                       float (&acc)[4][4]) {
  float a[4][8];
#pragma unroll
  for (int q = 0; q < 4; ++q) h8_to_f32(ar[q], a[q]);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float x[8];
    h8_to_f32(xr[i], x);
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int t = 0; t < 8; ++t) acc[i][q] = fmaf(x[t], a[q][t], acc[i][q]);
  }
}

// L2 prefetch of [p, p + bytes), one request per 128-byte line, spread over
// the CTA's threads; every address lies inside the range.
__device__ __forceinline__ void prefetch_l2(const void* p, int64_t bytes) {
  const char* c = static_cast<const char*>(p);
  for (int64_t off = (int64_t)threadIdx.x * 128; off < bytes; off += (int64_t)kLoraThreads * 128)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(c + off));
}

template <int R>
__global__ void __launch_bounds__(kLoraThreads, 2) lora_delta_kernel(
    const __half* __restrict__ X, const int32_t* __restrict__ offsets, int E, int N, int K, int r,
    const __half* __restrict__ lA, const __half* __restrict__ lB, float scale, int M_total,
    int nsplit, float* __restrict__ out, int32_t* dev_err) {
  __shared__ int s_off[kLoraMaxE + 1];
  __shared__ int tile_prefix[kLoraMaxE + 1];
  __shared__ int s_total;
  __shared__ __align__(16) float u[R][kLoraMaxRank];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  // offsets into shared memory in one pass, then tile_prefix[e] = sum over
  // e' < e of ceil(count_e' / R); offsets that are not monotone from 0 to
  // M_total void the launch (no output written)
  for (int i = threadIdx.x; i <= E; i += kLoraThreads) s_off[i] = offsets[i];
  __syncthreads();
  if (warp == 0) {
    bool bad = s_off[0] != 0 || s_off[E] != M_total;
    int run = 0;
    for (int b0 = 0; b0 < E; b0 += 32) {
      const int e = b0 + lane;
      int c = 0;
      if (e < E) {
        c = s_off[e + 1] - s_off[e];
        if (c < 0) { bad = true; c = 0; }
      }
      const int tiles = (c + R - 1) / R;
      int incl = tiles;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (e < E) tile_prefix[e] = run + incl - tiles;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      tile_prefix[E] = run;
      s_total = bad ? 0 : run;
      if (bad && blockIdx.x == 0) set_dev_err(dev_err, MOE_DEVERR_BAD_OFFSETS);
    }
  }
  __syncthreads();
  const int tile = blockIdx.x / nsplit, split = blockIdx.x % nsplit;
  if (tile >= s_total) return;

  // the expert whose tiles hold `tile`: the last e with tile_prefix[e] <= tile
  int lo = 0, hi = E;  // invariant: tile_prefix[lo] <= tile < tile_prefix[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tile_prefix[mid] <= tile) lo = mid; else hi = mid;
  }
  const int e = lo;
  const int row0 = s_off[e] + (tile - tile_prefix[e]) * R;
  const int nrows = min(R, s_off[e + 1] - row0);

  // Ask L2 for everything this CTA reads (the tile's input rows, A_e, its
  // columns of B_e and of the output rows) before the first demand load, so
  // that the dependent loads below meet L2 rather than HBM.
  const int cols = (N + nsplit - 1) / nsplit;
  const int n_begin = split * cols, n_end = min(N, n_begin + cols);
  const __half* Ae = lA + (int64_t)e * r * K;
  const __half* Be = lB + (int64_t)e * N * r;
  float* orow = out + (int64_t)row0 * N;
  prefetch_l2(X + (int64_t)row0 * K, (int64_t)nrows * K * 2);
  prefetch_l2(Ae, (int64_t)r * K * 2);
  if (n_begin < n_end) {
    prefetch_l2(Be + (int64_t)n_begin * r, (int64_t)(n_end - n_begin) * r * 2);
    for (int i = 0; i < nrows; ++i)
      prefetch_l2(orow + (int64_t)i * N + n_begin, (int64_t)(n_end - n_begin) * 4);
  }

  // ---- phase 1: u = A_e x for the tile's rows; the loads of the next
  // 256-wide k step are in flight while the current one is multiplied
  const int pblocks = (nrows + 3) >> 2, jblocks = r >> 2;
  for (int item = warp; item < pblocks * jblocks; item += kLoraWarps) {
    const int pb = item / jblocks, jb = item - pb * jblocks;
    const __half* xrow[4];
    const __half* arow[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // rows past the tile read row 0 of the tile (in range) and are dropped
      const int ri = pb * 4 + i < nrows ? pb * 4 + i : 0;
      xrow[i] = X + (int64_t)(row0 + ri) * K;
      arow[i] = Ae + (int64_t)(jb * 4 + i) * K;
    }
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[i][q] = 0.0f;
    int k = lane * 8;
    uint4 xr[4], ar[4];
    if (k < K) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        xr[i] = __ldg(reinterpret_cast<const uint4*>(xrow[i] + k));
        ar[i] = __ldg(reinterpret_cast<const uint4*>(arow[i] + k));
      }
    }
    for (; k < K; k += 256) {
      uint4 xn[4], an[4];
      const bool more = k + 256 < K;
      if (more) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          xn[i] = __ldg(reinterpret_cast<const uint4*>(xrow[i] + k + 256));
          an[i] = __ldg(reinterpret_cast<const uint4*>(arow[i] + k + 256));
        }
      }
      dot4x4(xr, ar, acc);
      if (more) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          xr[i] = xn[i];
          ar[i] = an[i];
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float s = warp_sum(acc[i][q]);
        if (lane == 0) u[pb * 4 + i][jb * 4 + q] = scale * s;
      }
  }
  __syncthreads();

  // ---- phase 2: out[p0 + i][n] += B_e[n] . u[i] (u holds scale * A_e x) over this split's
  // columns.  Every load of a column (its R outputs, its B_e row) comes
  // before the first store, so the loads overlap in one round trip.
  for (int n = n_begin + (int)threadIdx.x; n < n_end; n += kLoraThreads) {
    const __half* brow = Be + (int64_t)n * r;
    float o[R];
#pragma unroll
    for (int i = 0; i < R; ++i) o[i] = i < nrows ? orow[(int64_t)i * N + n] : 0.0f;
#pragma unroll
    for (int c = 0; c < kLoraMaxRank / 8; ++c) {
      if (c * 8 < r) {
        float b[8];
        h8_to_f32(__ldg(reinterpret_cast<const uint4*>(brow + c * 8)), b);
#pragma unroll
        for (int i = 0; i < R; ++i) {
          const float4 u0 = *reinterpret_cast<const float4*>(&u[i][c * 8]);
          const float4 u1 = *reinterpret_cast<const float4*>(&u[i][c * 8 + 4]);
          o[i] = fmaf(b[0], u0.x, o[i]);
          o[i] = fmaf(b[1], u0.y, o[i]);
          o[i] = fmaf(b[2], u0.z, o[i]);
          o[i] = fmaf(b[3], u0.w, o[i]);
          o[i] = fmaf(b[4], u1.x, o[i]);
          o[i] = fmaf(b[5], u1.y, o[i]);
          o[i] = fmaf(b[6], u1.z, o[i]);
          o[i] = fmaf(b[7], u1.w, o[i]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < R; ++i)
      if (i < nrows) orow[(int64_t)i * N + n] = o[i];
  }
}

}  // namespace
}  // namespace moe

namespace moe_launch {

bool lora_delta_supported(int E, int K, int r) {
  return E <= moe::kLoraMaxE && K % 8 == 0 && r >= 8 && r <= moe::kLoraMaxRank && r % 8 == 0;
}

cudaError_t lora_delta(const void* X, const int32_t* offsets, int E, int N, int K, int r,
                       const void* lora_A, const void* lora_B, float scale, int M_total,
                       float* out, int32_t* dev_err, cudaStream_t s) {
  if (M_total == 0) return cudaSuccess;
  // average rows per expert decides the tile height: 16 once the segments
  // are long enough to fill it, else 8
  const bool tall = (int64_t)M_total >= 16LL * E;
  const int R = tall ? 16 : 8;
  // every tile holds >= 1 row, and sum ceil(c / R) <= (M_total + E (R - 1)) / R
  const int64_t tiles = std::min<int64_t>(M_total, ((int64_t)M_total + (int64_t)E * (R - 1)) / R);
  // split the columns so that short launches still cover the SMs twice over,
  // never below 256 columns a split
  const int64_t want = (2LL * moe::device_sm_count() + tiles - 1) / tiles;
  const int nsplit = (int)std::max<int64_t>(1, std::min<int64_t>(want, std::max(1, N / 256)));
  const int64_t grid = tiles * nsplit;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  const __half* Xh = reinterpret_cast<const __half*>(X);
  const __half* Ah = reinterpret_cast<const __half*>(lora_A);
  const __half* Bh = reinterpret_cast<const __half*>(lora_B);
  if (tall)
    moe::lora_delta_kernel<16><<<(unsigned)grid, moe::kLoraThreads, 0, s>>>(
        Xh, offsets, E, N, K, r, Ah, Bh, scale, M_total, nsplit, out, dev_err);
  else
    moe::lora_delta_kernel<8><<<(unsigned)grid, moe::kLoraThreads, 0, s>>>(
        Xh, offsets, E, N, K, r, Ah, Bh, scale, M_total, nsplit, out, dev_err);
  return cudaGetLastError();
}

}  // namespace moe_launch
