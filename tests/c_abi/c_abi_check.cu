// GPU check through the C ABI alone: runs the MXFP4 quantize and decode GEMV
// and the backward kernels on inputs that make_inputs.py prepared (seeded
// numpy and the oracle), and writes every output as a raw file for
// compare.py to check against the oracle.
//   usage: c_abi_check <input dir> <output dir>   (both ending in '/')
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>
#include <cuda_runtime.h>
#include "moe_nf4.h"

static std::string IN, OUT;
static int fails = 0;
#define CK(x) do { cudaError_t e_ = (x); if (e_ != cudaSuccess) { printf("CUDA %s at %d\n", cudaGetErrorString(e_), __LINE__); exit(3); } } while (0)
#define ST(x) do { moe_status_t s_ = (x); if (s_ != MOE_OK) { printf("status %s at %d\n", moe_status_string(s_), __LINE__); fails++; } } while (0)

static void* load(const char* name, size_t bytes) {
  std::vector<char> h(bytes);
  FILE* f = fopen((IN + name).c_str(), "rb");
  if (!f || fread(h.data(), 1, bytes, f) != bytes) { printf("read %s failed\n", name); exit(2); }
  fclose(f);
  void* d; CK(cudaMalloc(&d, bytes < 16 ? 16 : bytes)); CK(cudaMemcpy(d, h.data(), bytes, cudaMemcpyHostToDevice));
  return d;
}
static void* zeros(size_t bytes) { void* d; CK(cudaMalloc(&d, bytes)); CK(cudaMemset(d, 0, bytes)); return d; }
static void dump(const char* name, const void* d, size_t bytes) {
  std::vector<char> h(bytes); CK(cudaMemcpy(h.data(), d, bytes, cudaMemcpyDeviceToHost));
  FILE* f = fopen((OUT + name).c_str(), "wb"); fwrite(h.data(), 1, bytes, f); fclose(f);
}
static int err_word(int32_t* d) { int v; CK(cudaMemcpy(&v, d, 4, cudaMemcpyDeviceToHost)); CK(cudaMemset(d, 0, 4)); return v; }

int main(int argc, char** argv) {
  if (argc != 3) { printf("usage: %s <input dir> <output dir>\n", argv[0]); return 2; }
  IN = argv[1];
  OUT = argv[2];
  int32_t* err = (int32_t*)zeros(4);
  // 1. MXFP4 quantize [3, 256, 768]
  { const int E = 3, N = 256, K = 768;
    float* W = (float*)load("mx_W.bin", (size_t)E * N * K * 4);
    uint8_t* P = (uint8_t*)zeros((size_t)E * N * K / 2); uint8_t* S = (uint8_t*)zeros((size_t)E * N * K / 32);
    ST(moe_mxfp4_quantize(W, E, N, K, P, S, err, nullptr)); CK(cudaDeviceSynchronize());
    printf("mxfp4_quantize dev_err=%d\n", err_word(err));
    dump("mxq_P.bin", P, (size_t)E * N * K / 2); dump("mxq_S.bin", S, (size_t)E * N * K / 32); }
  // 2. MXFP4 GEMV [6, 384, 512], M = 83, none / swiglu, fp32 out
  { const int E = 6, N = 384, K = 512, M = 83;
    void* P = load("mx_P.bin", (size_t)E * N * K / 2); void* S = load("mx_S.bin", (size_t)E * N * K / 32);
    void* X = load("mx_X.bin", (size_t)M * K * 2); int32_t* off = (int32_t*)load("mx_off.bin", (E + 1) * 4);
    float* o1 = (float*)zeros((size_t)M * N * 4); float* o2 = (float*)zeros((size_t)M * N / 2 * 4);
    ST(moe_mxfp4_grouped_gemm(X, M, (uint8_t*)P, (uint8_t*)S, off, E, N, K, M, MOE_EPI_NONE, o1, MOE_DT_F32, MOE_ALGO_GEMV, err, nullptr));
    ST(moe_mxfp4_grouped_gemm(X, M, (uint8_t*)P, (uint8_t*)S, off, E, N, K, M, MOE_EPI_SWIGLU, o2, MOE_DT_F32, MOE_ALGO_GEMV, err, nullptr));
    CK(cudaDeviceSynchronize());
    printf("mxfp4_gemm dev_err=%d\n", err_word(err));
    dump("mxg_none.bin", o1, (size_t)M * N * 4); dump("mxg_swiglu.bin", o2, (size_t)M * N / 2 * 4); }
  // 3. transposed NF4 GEMM [4, 2048, 1024], M = 56, G rows 58; and [4, 70, 320], M = 13
  { const int E = 4, N = 2048, K = 1024, M = 56;
    void* P = load("gt_P.bin", (size_t)E * N * K / 2); void* A = load("gt_A.bin", (size_t)E * N * K / 64 * 4);
    void* G = load("gt_G.bin", (size_t)(M + 2) * N * 4); int32_t* off = (int32_t*)load("gt_off.bin", (E + 1) * 4);
    float* o = (float*)zeros((size_t)M * K * 4);
    ST(moe_nf4_grouped_gemm_t(G, MOE_DT_F32, M + 2, (uint8_t*)P, (float*)A, off, E, N, K, M, o, MOE_DT_F32, MOE_ALGO_GEMV, err, nullptr));
    CK(cudaDeviceSynchronize()); printf("gemm_t dev_err=%d\n", err_word(err)); dump("gt_out.bin", o, (size_t)M * K * 4); }
  { const int E = 4, N = 70, K = 320, M = 13;
    void* P = load("gt2_P.bin", (size_t)E * N * K / 2); void* A = load("gt2_A.bin", (size_t)E * N * K / 64 * 4);
    void* G = load("gt2_G.bin", (size_t)M * N * 4); int32_t* off = (int32_t*)load("gt2_off.bin", (E + 1) * 4);
    float* o = (float*)zeros((size_t)M * K * 4);
    ST(moe_nf4_grouped_gemm_t(G, MOE_DT_F32, M, (uint8_t*)P, (float*)A, off, E, N, K, M, o, MOE_DT_F32, MOE_ALGO_GEMV, err, nullptr));
    CK(cudaDeviceSynchronize()); printf("gemm_t2 dev_err=%d\n", err_word(err)); dump("gt2_out.bin", o, (size_t)M * K * 4); }
  // 4. SwiGLU backward [37, 96]
  { const int M = 37, I = 96;
    void* gu = load("sb_gu.bin", (size_t)M * 2 * I * 4); void* dh = load("sb_dh.bin", (size_t)M * I * 4);
    float* o = (float*)zeros((size_t)M * 2 * I * 4);
    ST(moe_swiglu_backward(gu, dh, MOE_DT_F32, M, I, o, MOE_DT_F32, nullptr));
    CK(cudaDeviceSynchronize()); dump("sb_out.bin", o, (size_t)M * 2 * I * 4); }
  // 5. combine + route backward, T 33, E 16, k 4, H 256, renorm 0 / 1
  { const int T = 33, E = 16, k = 4, H = 256;
    float* lg = (float*)load("cb_lg.bin", (size_t)T * E * 4); void* Yp = load("cb_Yp.bin", (size_t)T * k * H * 4);
    float* dY = (float*)load("cb_dY.bin", (size_t)T * H * 4);
    for (int rn = 0; rn < 2; ++rn) {
      char nm[64];
      snprintf(nm, 64, "cb_idx%d.bin", rn); int32_t* idx = (int32_t*)load(nm, (size_t)T * k * 4);
      snprintf(nm, 64, "cb_w%d.bin", rn); float* w = (float*)load(nm, (size_t)T * k * 4);
      snprintf(nm, 64, "cb_inv%d.bin", rn); int32_t* inv = (int32_t*)load(nm, (size_t)T * k * 4);
      float* dYp = (float*)zeros((size_t)T * k * H * 4); float* dw = (float*)zeros((size_t)T * k * 4);
      float* dl = (float*)zeros((size_t)T * E * 4);
      ST(moe_combine_backward(dY, Yp, MOE_DT_F32, inv, w, T, k, H, dYp, MOE_DT_F32, dw, err, nullptr));
      ST(moe_route_backward(lg, idx, w, dw, T, E, k, rn, dl, err, nullptr));
      CK(cudaDeviceSynchronize()); printf("combine/route bw rn=%d dev_err=%d\n", rn, err_word(err));
      snprintf(nm, 64, "cb_dYp%d.bin", rn); dump(nm, dYp, (size_t)T * k * H * 4);
      snprintf(nm, 64, "cb_dw%d.bin", rn); dump(nm, dw, (size_t)T * k * 4);
      snprintf(nm, 64, "cb_dl%d.bin", rn); dump(nm, dl, (size_t)T * E * 4);
    } }
  printf("done fails=%d\n", fails);
  return fails ? 1 : 0;
}
