// Backward of the layer with the 4-bit experts frozen: the transposed grouped
// NF4 GEMM, SwiGLU backward, combine backward and routing backward.
//
// The pages' kernel is differentiable and fine-tunes on the packed 4-bit
// weights without unpacking them; the frozen stack stays byte-identical
// ("Jordan Anderson", jordananderson-pages.pages.dev, section "grouped-nf4-gemm
// & experts-4bit", fourth bullet).  The gradients are the chain rule through
// the forward layer:
//   transposed GEMM   dX[p] = W[e(p)]^T g[p]  (the weights' NF4 blocks now run
//                     along the OUTPUT dimension, so each output column keeps
//                     one absmax per weight row)
//   SwiGLU            s = sigmoid(g); dg = dh u s (1 + g (1 - s)), du = dh g s
//   combine           dYp[pos(t,j)] = w[t,j] dY[t]; dw[t,j] = <dY[t], Yp[pos(t,j)]>
//   routing           renormalised: dl[e_j] = w_j (dw_j - sum_j' dw_j' w_j');
//                     plain softmax: dl_i = [i = e_j] dw_j w_j - p_i sum_j dw_j w_j
// The scatter-add of routed-row gradients into tokens is moe_unpermute_combine
// with unit weights.
//
// First versions on the CUDA cores (fp32 FMA): the transposed GEMM streams each
// selected expert's packed bytes once per tile of up to 8 routed rows, 128
// consecutive bytes of a weight row per CTA row step (coalesced), decoding each
// byte through a 16-entry shared table and its row's absmax.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kBwThreads = 256;
constexpr int kTR = 8;        // routed rows per tile
constexpr int kTNC = 64;      // weight rows of g staged per step
constexpr int kTCols = 256;   // output columns per CTA (128 packed bytes)
constexpr int kMaxE = 1024;

template <typename T>
__device__ __forceinline__ float ld_f32(const T* p) {
  return to_f32<T>(*p);
}

template <typename GT, typename OutT>
__global__ void __launch_bounds__(kBwThreads) nf4_gemm_t_kernel(
    const GT* __restrict__ G, const uint8_t* __restrict__ packed,
    const float* __restrict__ absmax, const int32_t* __restrict__ offsets, int E, int N, int K,
    int M_total, int kchunks, OutT* __restrict__ out, int32_t* dev_err) {
  __shared__ int s_off[kMaxE + 1];
  __shared__ int tile_prefix[kMaxE + 1];
  __shared__ int s_total;
  __shared__ float lut[16];
  __shared__ float gs[kTR][kTNC];
  __shared__ __align__(8) float red[kTR][kTCols];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  for (int i = threadIdx.x; i <= E; i += kBwThreads) s_off[i] = offsets[i];
  if (threadIdx.x < 16) {
    const float levels[16] = {MOE_NF4_LEVEL_LIST};
    lut[threadIdx.x] = levels[threadIdx.x];
  }
  __syncthreads();
  if (warp == 0) {
    // tile_prefix[e] = sum over e' < e of ceil(count_e' / kTR); offsets that
    // are not monotone from 0 to M_total void the launch
    bool bad = s_off[0] != 0 || s_off[E] != M_total;
    int run = 0;
    for (int b0 = 0; b0 < E; b0 += 32) {
      const int e = b0 + lane;
      int c = 0;
      if (e < E) {
        c = s_off[e + 1] - s_off[e];
        if (c < 0) { bad = true; c = 0; }
      }
      const int tiles = (c + kTR - 1) / kTR;
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
  const int tile = blockIdx.x / kchunks, kc = blockIdx.x % kchunks;
  if (tile >= s_total) return;
  int lo = 0, hi = E;  // invariant: tile_prefix[lo] <= tile < tile_prefix[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tile_prefix[mid] <= tile) lo = mid; else hi = mid;
  }
  const int e = lo;
  const int row0 = s_off[e] + (tile - tile_prefix[e]) * kTR;
  const int nrows = min(kTR, s_off[e + 1] - row0);

  // thread (c, h): packed byte c of the chunk (output columns 2c, 2c+1),
  // weight rows n = h (mod 2)
  const int c = threadIdx.x & 127, h = threadIdx.x >> 7;
  const int half_k = K / 2;
  const int byte = kc * (kTCols / 2) + c;
  const bool col_ok = byte < half_k;
  const int kblocks = K / kBlock;
  const int kb = (2 * byte) / kBlock;  // NF4 block of this thread's columns
  const uint8_t* wcol = packed + (size_t)e * N * half_k + (col_ok ? byte : 0);
  const float* acol = absmax + (size_t)e * N * kblocks + (col_ok ? kb : 0);

  float acc[kTR][2];
#pragma unroll
  for (int p = 0; p < kTR; ++p) acc[p][0] = acc[p][1] = 0.0f;

  for (int n0 = 0; n0 < N; n0 += kTNC) {
    for (int i = threadIdx.x; i < kTR * kTNC; i += kBwThreads) {
      const int p = i / kTNC, j = i - p * kTNC;
      gs[p][j] = (p < nrows && n0 + j < N) ? ld_f32(G + (size_t)(row0 + p) * N + n0 + j) : 0.0f;
    }
    __syncthreads();
    const int jn = min(kTNC, N - n0);
#pragma unroll 8
    for (int j = h; j < jn; j += 2) {
      const size_t n = (size_t)(n0 + j);
      const uint32_t b = col_ok ? __ldg(wcol + n * half_k) : 0u;
      const float am = col_ok ? __ldg(acol + n * kblocks) : 0.0f;
      // NF4: element 2j of a row is the byte's high nibble
      const float v0 = lut[b >> 4] * am, v1 = lut[b & 15u] * am;
#pragma unroll
      for (int p = 0; p < kTR; ++p) {
        acc[p][0] = fmaf(v0, gs[p][j], acc[p][0]);
        acc[p][1] = fmaf(v1, gs[p][j], acc[p][1]);
      }
    }
    __syncthreads();
  }

  // the two row phases meet in shared memory; phase 0 writes the columns
  if (h == 1) {
#pragma unroll
    for (int p = 0; p < kTR; ++p)
      *reinterpret_cast<float2*>(&red[p][2 * c]) = make_float2(acc[p][0], acc[p][1]);
  }
  __syncthreads();
  if (h == 0 && col_ok) {
    for (int p = 0; p < nrows; ++p) {
      const float2 o = *reinterpret_cast<const float2*>(&red[p][2 * c]);
      OutT* dst = out + (size_t)(row0 + p) * K + 2 * byte;
      dst[0] = from_f32<OutT>(acc[p][0] + o.x);
      dst[1] = from_f32<OutT>(acc[p][1] + o.y);
    }
  }
}

template <typename InT, typename OutT>
__global__ void __launch_bounds__(256) swiglu_backward_kernel(const InT* __restrict__ gu,
                                                              const InT* __restrict__ dh, int M,
                                                              int I, OutT* __restrict__ dgu) {
  const int64_t total = (int64_t)M * I;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < total; q += stride) {
    const int64_t m = q / I, i = q - m * I;
    const float g = to_f32<InT>(gu[m * 2 * I + i]);
    const float u = to_f32<InT>(gu[m * 2 * I + I + i]);
    const float d = to_f32<InT>(dh[m * I + i]);
    const float s = __fdiv_rn(1.0f, 1.0f + expf(-g));
    const float dsilu = s * (1.0f + g * (1.0f - s));
    dgu[m * 2 * I + i] = from_f32<OutT>(d * u * dsilu);
    dgu[m * 2 * I + I + i] = from_f32<OutT>(d * g * s);
  }
}

// one warp per routed row (t, j)
template <typename YT, typename OutT>
__global__ void __launch_bounds__(256) combine_backward_kernel(
    const float* __restrict__ dY, const YT* __restrict__ Yp, const int32_t* __restrict__ inv_perm,
    const float* __restrict__ w, int T, int k, int H, OutT* __restrict__ dYp,
    float* __restrict__ dw, int32_t* dev_err) {
  const int lane = threadIdx.x & 31;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t total = (int64_t)T * k;
  for (int64_t f = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; f < total; f += nw) {
    const int t = (int)(f / k);
    const int pos = inv_perm[f];
    if (pos < 0 || pos >= total) {
      if (lane == 0) {
        set_dev_err(dev_err, MOE_DEVERR_BAD_INDEX);
        dw[f] = 0.0f;
      }
      continue;
    }
    const float wt = w[f];
    float dot = 0.0f;
    for (int c = lane; c < H; c += 32) {
      const float d = dY[(size_t)t * H + c];
      dot = fmaf(d, to_f32<YT>(Yp[(size_t)pos * H + c]), dot);
      dYp[(size_t)pos * H + c] = from_f32<OutT>(wt * d);
    }
    dot = warp_sum(dot);
    if (lane == 0) dw[f] = dot;
  }
}

// one warp per token
__global__ void __launch_bounds__(256) route_backward_kernel(
    const float* __restrict__ logits, const int32_t* __restrict__ idx,
    const float* __restrict__ w, const float* __restrict__ dw, int T, int E, int k,
    int renormalize, float* __restrict__ dl, int32_t* dev_err) {
  const int lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nw) {
    const float* lt = logits + (size_t)t * E;
    float* out = dl + (size_t)t * E;
    // c = sum_j dw_j w_j over the k selected experts (k <= 32: one per lane)
    float wj = 0.0f, dwj = 0.0f;
    int ej = -1;
    if (lane < k) {
      ej = idx[(size_t)t * k + lane];
      wj = w[(size_t)t * k + lane];
      dwj = dw[(size_t)t * k + lane];
      if (ej < 0 || ej >= E) {
        set_dev_err(dev_err, MOE_DEVERR_BAD_INDEX);
        ej = -1;
      }
    }
    const float cs = warp_sum(dwj * wj);
    if (renormalize) {
      for (int i = lane; i < E; i += 32) out[i] = 0.0f;
    } else {
      float m = -INFINITY;
      for (int i = lane; i < E; i += 32) m = fmaxf(m, lt[i]);
      m = warp_max(m);
      float z = 0.0f;
      for (int i = lane; i < E; i += 32) z += expf(lt[i] - m);
      z = warp_sum(z);
      for (int i = lane; i < E; i += 32) out[i] = -__fdiv_rn(expf(lt[i] - m), z) * cs;
    }
    __syncwarp();
    // the selected experts are distinct, so each lane owns its entry
    if (ej >= 0) {
      if (renormalize) out[ej] = wj * (dwj - cs);
      else out[ej] += dwj * wj;
    }
    __syncwarp();
  }
}

int sm_count() { return device_sm_count(); }

template <typename GT, typename OutT>
cudaError_t gemm_t_launch(const void* G, const uint8_t* packed, const float* absmax,
                          const int32_t* offsets, int E, int N, int K, int M_total, void* out,
                          int32_t* dev_err, cudaStream_t s) {
  const int64_t tiles =
      std::min<int64_t>(M_total, ((int64_t)M_total + (int64_t)E * (kTR - 1)) / kTR);
  const int kchunks = (K + kTCols - 1) / kTCols;
  const int64_t grid = tiles * kchunks;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  nf4_gemm_t_kernel<GT, OutT><<<(unsigned)grid, kBwThreads, 0, s>>>(
      reinterpret_cast<const GT*>(G), packed, absmax, offsets, E, N, K, M_total, kchunks,
      reinterpret_cast<OutT*>(out), dev_err);
  return cudaGetLastError();
}

}  // namespace
}  // namespace moe

namespace moe_launch {

cudaError_t grouped_gemm_t(const void* G, moe_dtype_t g_dt, const uint8_t* packed,
                           const float* absmax, const int32_t* offsets, int E, int N, int K,
                           int M_total, void* out, moe_dtype_t out_dt, int32_t* dev_err,
                           cudaStream_t s) {
  using namespace moe;
  if (M_total == 0) return cudaSuccess;
  if (g_dt == MOE_DT_F32) {
    if (out_dt == MOE_DT_F32)
      return gemm_t_launch<float, float>(G, packed, absmax, offsets, E, N, K, M_total, out,
                                         dev_err, s);
    return gemm_t_launch<float, __half>(G, packed, absmax, offsets, E, N, K, M_total, out,
                                        dev_err, s);
  }
  if (out_dt == MOE_DT_F32)
    return gemm_t_launch<__half, float>(G, packed, absmax, offsets, E, N, K, M_total, out,
                                        dev_err, s);
  return gemm_t_launch<__half, __half>(G, packed, absmax, offsets, E, N, K, M_total, out, dev_err,
                                       s);
}

cudaError_t swiglu_backward(const void* gu, const void* dh, moe_dtype_t in_dt, int M, int I,
                            void* dgu, moe_dtype_t out_dt, cudaStream_t s) {
  using namespace moe;
  const int64_t total = (int64_t)M * I;
  if (total == 0) return cudaSuccess;
  const int grid = (int)std::min<int64_t>((total + 255) / 256, (int64_t)sm_count() * 8);
#define MOE_SWB(IT, OT)                                                                        \
  swiglu_backward_kernel<IT, OT><<<grid, 256, 0, s>>>(reinterpret_cast<const IT*>(gu),         \
                                                      reinterpret_cast<const IT*>(dh), M, I,   \
                                                      reinterpret_cast<OT*>(dgu))
  if (in_dt == MOE_DT_F32) {
    if (out_dt == MOE_DT_F32) MOE_SWB(float, float);
    else MOE_SWB(float, __half);
  } else {
    if (out_dt == MOE_DT_F32) MOE_SWB(__half, float);
    else MOE_SWB(__half, __half);
  }
#undef MOE_SWB
  return cudaGetLastError();
}

cudaError_t combine_backward(const float* dY, const void* Yp, moe_dtype_t yp_dt,
                             const int32_t* inv_perm, const float* topk_w, int T, int k, int H,
                             void* dYp, moe_dtype_t dyp_dt, float* dw, int32_t* dev_err,
                             cudaStream_t s) {
  using namespace moe;
  const int64_t rows = (int64_t)T * k;
  if (rows == 0) return cudaSuccess;
  const int grid = (int)std::min<int64_t>((rows + 7) / 8, (int64_t)sm_count() * 16);
#define MOE_CBB(YT, OT)                                                                          \
  combine_backward_kernel<YT, OT><<<grid, 256, 0, s>>>(dY, reinterpret_cast<const YT*>(Yp),      \
                                                       inv_perm, topk_w, T, k, H,                \
                                                       reinterpret_cast<OT*>(dYp), dw, dev_err)
  if (yp_dt == MOE_DT_F32) {
    if (dyp_dt == MOE_DT_F32) MOE_CBB(float, float);
    else MOE_CBB(float, __half);
  } else {
    if (dyp_dt == MOE_DT_F32) MOE_CBB(__half, float);
    else MOE_CBB(__half, __half);
  }
#undef MOE_CBB
  return cudaGetLastError();
}

cudaError_t route_backward(const float* logits, const int32_t* topk_idx, const float* topk_w,
                           const float* dw, int T, int E, int k, int renormalize, float* dlogits,
                           int32_t* dev_err, cudaStream_t s) {
  using namespace moe;
  if (T == 0) return cudaSuccess;
  const int grid = (int)std::min<int64_t>(((int64_t)T + 7) / 8, (int64_t)sm_count() * 16);
  route_backward_kernel<<<grid, 256, 0, s>>>(logits, topk_idx, topk_w, dw, T, E, k, renormalize,
                                             dlogits, dev_err);
  return cudaGetLastError();
}

}  // namespace moe_launch
