/*
 * moe_nf4.h -- C ABI of the B200 (sm_100a) NF4 grouped mixture-of-experts
 * library (libmoenf4.so).
 *
 * The library runs one mixture-of-experts layer directly on 4-bit NF4 expert
 * weights: top-k routing and a token->expert permutation, one grouped GEMM
 * launch over all active experts for gate_up with SiLU(gate)*up fused in its
 * epilogue, a grouped down projection, and a routing-weighted combine.  The
 * NF4 codebook and per-block absmax are decoded in registers inside the GEMM;
 * no dequantized weight copy is ever written to memory.  The method is the
 * one described in "grouped-nf4-gemm & experts-4bit" (jordananderson-pages
 * .pages.dev), first bullet, and in the "grouped-nf4-gemm" bullet of the
 * pjordanandrsn GitHub profile page.
 *
 * Beyond the NF4 forward: the same grouped GEMV on GPTQ-style INT4 and on
 * MXFP4 weights, a per-expert LoRA delta, and the backward steps of the layer
 * with the 4-bit experts frozen (transposed grouped GEMM, SwiGLU, combine and
 * routing backward).
 *
 * Conventions shared by every call
 * --------------------------------
 * - All pointers are DEVICE pointers unless a parameter says otherwise; the
 *   caller allocates and owns every buffer (inputs, outputs, workspace); the
 *   library allocates no device memory.  It does keep process-wide state of
 *   two kinds: (1) host-side caches -- encoded TMA tensor maps, keyed by
 *   every argument that determines them, and per-device attributes -- which
 *   never change a result; (2) the fixed scratch array of
 *   moe_route_permute_noalloc (see there).
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream).  Every call only enqueues work: it is asynchronous and
 *   stream-ordered, and never synchronizes the device.
 * - Matrices are dense and row-major.  Sizes are element counts.
 * - Synchronous argument errors return at once and enqueue nothing.
 *   A launch failure returns MOE_ERR_CUDA.  Contract violations that only
 *   the device can see (non-finite weights, inconsistent expert offsets,
 *   an expert index out of range) set a bit in the caller's device word
 *   `dev_err` (int32, may be NULL) and the affected work is skipped; the
 *   caller reads the word when it chooses.  No kernel traps or asserts.
 * - sm_100a only: calls on another architecture return MOE_ERR_UNSUPPORTED.
 *
 * NF4 weight layout (the fused 3-D expert parameter of "4-bit
 * Mixture-of-Experts fine-tuning on small GPUs", jordananderson.work, first
 * bullet, quantized as in "grouped-nf4-gemm & experts-4bit", first bullet):
 * - a stack of E experts, each an [N, K] out x in matrix, K % 64 == 0;
 * - packed  uint8 [E, N, K/2]: element 2j of a row in the HIGH nibble of
 *   byte j, element 2j+1 in the low nibble;
 * - absmax  fp32  [E, N*K/64]: one scale per 64 consecutive elements of a
 *   row; weight = NF4_LEVEL[code] * absmax.
 * gate_up stacks are [E, 2I, H] with rows [0, I) the gate and [I, 2I) the
 * up projection; down stacks are [E, H, I].
 */
#ifndef MOE_NF4_H
#define MOE_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_NF4_ABI_VERSION 3

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, bad size or enum value       */
  MOE_ERR_MISALIGNED = 2,  /* a pointer is not 16-byte aligned           */
  MOE_ERR_UNSUPPORTED = 3, /* shape or device this build does not cover  */
  MOE_ERR_WORKSPACE = 4,   /* workspace missing or too small             */
  MOE_ERR_CUDA = 5         /* a CUDA launch or runtime call failed       */
} moe_status_t;

typedef enum { MOE_DT_F32 = 0, MOE_DT_BF16 = 1, MOE_DT_F16 = 2 } moe_dtype_t;

typedef enum { MOE_EPI_NONE = 0, MOE_EPI_SWIGLU = 1 } moe_epilogue_t;

/* Grouped-GEMM kernel choice.  AUTO picks GEMV for small row counts and the
 * tensor-memory (tcgen05) kernel otherwise; the others force one path. */
typedef enum {
  MOE_ALGO_AUTO = 0,
  MOE_ALGO_GEMV = 1,    /* decode: streams weights, warp MMA per 16 rows    */
  MOE_ALGO_TC = 2,      /* prefill: tcgen05.mma with TMEM accumulators, one
                           CTA per 128-weight-row tile                      */
  MOE_ALGO_TC_PAIR = 3  /* the same on CTA pairs (cta_group::2, M = 256, two
                           SMs per 256-weight-row tile); needs N % 256 == 0.
                           Measured slower than MOE_ALGO_TC on the Qwen3
                           shapes, so AUTO does not pick it                 */
} moe_algo_t;

/* Bits the kernels OR into the caller's device error word. */
#define MOE_DEVERR_NONFINITE 0x1   /* quantize saw a NaN or Inf weight      */
#define MOE_DEVERR_BAD_OFFSETS 0x2 /* expert_offsets not monotone / total   */
#define MOE_DEVERR_BAD_INDEX 0x4   /* a row or expert index out of range    */
#define MOE_DEVERR_TIMEOUT 0x8     /* a bounded wait inside a kernel expired */
#define MOE_DEVERR_LAYOUT 0x10     /* a kernel's shared-memory layout did not
                                      fit this device; the call did no work */
#define MOE_DEVERR_RANGE 0x20      /* a value outside the range of the 16-bit
                                      type it passes through: an fp16
                                      activation, intermediate or output
                                      that overflowed; an NF4 absmax that is
                                      subnormal or too large in fp16 (tensor-
                                      core GEMM); an MXFP4 scale outside the
                                      range the decode GEMV multiplies
                                      exactly.  The work is done; the
                                      affected values carry the error */

/* Human-readable name of a status code (static string, never NULL). */
const char* moe_status_string(moe_status_t status);

/* MOE_NF4_ABI_VERSION of the loaded library. */
int moe_abi_version(void);

/* Text of the CUDA error behind the calling host thread's most recent
 * MOE_ERR_CUDA ("no error" if none); a static string, never NULL. */
const char* moe_last_cuda_error(void);

/* Copies the library's 16 NF4 levels (fp32, ascending, code c -> level c)
 * into HOST memory `levels_out[16]`.  Host-only, no CUDA call. */
moe_status_t moe_nf4_levels(float* levels_out);

/*
 * moe_nf4_quantize -- blockwise NF4 quantization of a fused expert stack.
 * ("4-bit Mixture-of-Experts fine-tuning on small GPUs", jordananderson.work,
 * second bullet: the primitive that quantizes the fused expert stack.)
 *
 *   W       fp32  [E, N, K]    input weights (device, read only)
 *   E, N, K >= 1, K % 64 == 0
 *   blocksize must be 64
 *   packed  uint8 [E, N, K/2]  output codes (device)
 *   absmax  fp32  [E, N*K/64]  output scales (device)
 *   dev_err int32 device word or NULL; MOE_DEVERR_NONFINITE is set if any
 *           weight is NaN/Inf (its block's codes are then unspecified).
 * Per 64-block: a = max|x|; a == 0 -> every code 7; else n = x / a (IEEE
 * fp32 division) and code = #{i : n > fl32(L_i + L_{i+1}) * 0.5}, i.e. the
 * nearest level with ties to the lower code.  Deterministic, bit-exact.
 * W, packed and absmax must be 16-byte aligned.
 */
moe_status_t moe_nf4_quantize(const float* W, int E, int N, int K,
                              int blocksize, uint8_t* packed, float* absmax,
                              int32_t* dev_err, void* stream);

/*
 * Inverse of the quantizer for inspection and tests: out[E, N, K] =
 * L[code] * absmax, the exact product rounded once to `out_dtype`.
 */
moe_status_t moe_nf4_dequantize(const uint8_t* packed, const float* absmax,
                                int E, int N, int K, void* out,
                                moe_dtype_t out_dtype, void* stream);

/*
 * moe_int4_quantize -- grouped INT4 quantization of a fused expert stack, the
 * format of moe_int4_grouped_gemm.  ("grouped-nf4-gemm & experts-4bit",
 * jordananderson-pages.pages.dev, third bullet: GPTQ-calibrated int4 experts
 * served by an INT4 decode GEMV.  The pages fix no format; this one follows
 * the GPTQ checkpoint convention.)
 *
 *   W       fp32   [E, N, K]      input weights (device, read only)
 *   E, N, K >= 1, K % 128 == 0
 *   packed  uint8  [E, N, K/2]    codes q, two per byte, element 2j of a row in
 *                                 the high nibble of byte j (device)
 *   meta    uint32 [E, N, K/128]  per group of 128 along K: fp16 bits of the
 *                                 scale s | zero z << 16 (device)
 *   dev_err int32 device word or NULL; MOE_DEVERR_NONFINITE if any weight is
 *           NaN/Inf (its group's codes are then unspecified).
 * Per group: lo = min(min x, 0), hi = max(max x, 0), s = fp16(fl32((hi-lo)/15)),
 * z = clamp(rint(-lo/s), 0, 15), q = clamp(rint(x/s) + z, 0, 15) (IEEE fp32
 * division, rint to nearest even); stored scale 0 -> z = 0, q = 0.  The value
 * of a code is (q - z) * s.  Round-to-nearest, deterministic, bit-exact.
 * W, packed and meta must be 16-byte aligned.
 */
moe_status_t moe_int4_quantize(const float* W, int E, int N, int K, uint8_t* packed,
                               uint32_t* meta, int32_t* dev_err, void* stream);

/*
 * moe_int4_grouped_gemm -- grouped GEMM on INT4 weights:
 * out[p] = W[e(p)] @ A[p] for every row p in expert e's segment
 * [expert_offsets[e], expert_offsets[e+1]), W[e] = (q - z) * s from
 * (packed, meta) as written by moe_int4_quantize, all experts in one launch.
 *
 *   A        fp16 [A_rows >= M_total, K]  routed rows in permuted order
 *            (e.g. moe_permute_rows output); no gather
 *   packed   uint8 [E, N, K/2], meta uint32 [E, N, K/128]
 *   expert_offsets int32 [E+1] (device), monotone, offsets[E] == M_total
 *   E <= 1024; decode GEMV: N % 128 == 0, K % 256 == 0; tensor-core kernel:
 *            N % 128 == 0, K % 128 == 0
 *   epilogue MOE_EPI_NONE: out [M_total, N]; MOE_EPI_SWIGLU: rows [0, N/2)
 *            are gate and [N/2, N) up, out [M_total, N/2] = silu(g) * u
 *   out      F32 / F16 / BF16
 *   algo     AUTO: the tensor-core kernel from 36 routed rows per expert on
 *            average (as the NF4 call), else the decode GEMV; GEMV / TC force
 *   dev_err  as moe_nf4_grouped_gemm (BAD_OFFSETS, TIMEOUT, LAYOUT, RANGE)
 * Decode GEMV: the weights enter the MMA as the exact integers q - z (fp16);
 * each 64-k block's fp32 partial sum is scaled by its group's s.  Streams
 * every selected expert's bytes once (HBM-bound at decode sizes).
 * Tensor-core kernel (tcgen05): weights enter as fp16((q - z) * s), one
 * rounding of the exact value; sums fp32 in TMEM.
 * All pointers 16-byte aligned.
 */
moe_status_t moe_int4_grouped_gemm(const void* A, int A_rows, const uint8_t* packed,
                                   const uint32_t* meta, const int32_t* expert_offsets, int E,
                                   int N, int K, int M_total, moe_epilogue_t epilogue, void* out,
                                   moe_dtype_t out_dtype, moe_algo_t algo, int32_t* dev_err,
                                   void* stream);

/*
 * moe_mxfp4_quantize -- MXFP4 quantization of a fused expert stack, the format
 * of moe_mxfp4_grouped_gemm.  ("grouped-nf4-gemm & experts-4bit",
 * jordananderson-pages.pages.dev, third bullet: the kernel serves MXFP4 on a
 * checkpoint's released bytes; e2m1 + e8m0 per "MoE Training on Consumer
 * GPUs", cerinamroth.com/ml.  Format and conversion: OCP Microscaling v1.0.)
 *
 *   W       fp32   [E, N, K]      input weights (device, read only)
 *   E, N, K >= 1, K % 32 == 0
 *   packed  uint8  [E, N, K/2]    E2M1 codes, two per byte, element 2j of a
 *                                 row in the LOW nibble of byte j (device)
 *   scales  uint8  [E, N, K/32]   E8M0 byte b per 32 along K, 2^(b - 127)
 *   dev_err int32 device word or NULL; MOE_DEVERR_NONFINITE if any weight is
 *           NaN/Inf (its block's bytes are then unspecified).
 * Per block: shared = clamp(floor(log2 max|x|) - 2, -127, 127), b = shared +
 * 127; codes = nearest E2M1 value of x * 2^-shared (exact in fp32), ties to
 * the even mantissa, saturating at +-6, a value rounding to zero -> code 0;
 * an all-zero block -> b = 0, codes 0.  Deterministic, bit-exact.
 * W, packed and scales must be 16-byte aligned.
 */
moe_status_t moe_mxfp4_quantize(const float* W, int E, int N, int K, uint8_t* packed,
                                uint8_t* scales, int32_t* dev_err, void* stream);

/*
 * moe_mxfp4_grouped_gemm -- grouped GEMM on MXFP4 weights:
 * out[p] = W[e(p)] @ A[p] for every row p in expert e's segment
 * [expert_offsets[e], expert_offsets[e+1]), W[e] = 2^(b - 127) * e2m1(code)
 * from (packed, scales) as written by moe_mxfp4_quantize or taken unchanged
 * from a released MXFP4 checkpoint in this layout, all experts in one launch.
 *
 *   A        fp16 [A_rows >= M_total, K]  routed rows in permuted order
 *   packed   uint8 [E, N, K/2], scales uint8 [E, N, K/32]
 *   expert_offsets int32 [E+1] (device), monotone, offsets[E] == M_total
 *   E <= 1024; GEMV kernel: N % 128 == 0, K % 256 == 0; tensor-core kernel:
 *            N % 128 == 0, K % 64 == 0
 *   epilogue MOE_EPI_NONE: out [M_total, N]; MOE_EPI_SWIGLU: rows [0, N/2)
 *            are gate and [N/2, N) up, out [M_total, N/2] = silu(g) * u
 *   out      F32 / F16 / BF16
 *   algo     AUTO takes the tensor-core kernel (tcgen05, TMEM accumulators)
 *            from 36 routed rows per expert on average, as the NF4 call does,
 *            else the decode GEMV; GEMV / TC force one
 *   dev_err  BAD_OFFSETS, TIMEOUT, LAYOUT as moe_nf4_grouped_gemm; RANGE when
 *            a scale byte is neither 0 nor in [104, 140], where the weights
 *            are not exact in fp16 (products then rounded or flushed), or an
 *            fp16 output overflowed
 * Both kernels feed the weights to the tensor cores as exact fp16 values
 * (E2M1 times the scale's power of two) with fp16 activations; sums are fp32.
 * (Blackwell's block-scaled kind::mxf4 MMA would take the codes and scales
 * directly, but it needs the activations in FP4 or FP8 as well, which puts
 * the layer outside the parity tolerance; see the design notes.)
 * All pointers 16-byte aligned.
 */
moe_status_t moe_mxfp4_grouped_gemm(const void* A, int A_rows, const uint8_t* packed,
                                    const uint8_t* scales, const int32_t* expert_offsets, int E,
                                    int N, int K, int M_total, moe_epilogue_t epilogue, void* out,
                                    moe_dtype_t out_dtype, moe_algo_t algo, int32_t* dev_err,
                                    void* stream);

/*
 * Backward of the layer with the 4-bit experts frozen ("grouped-nf4-gemm &
 * experts-4bit", jordananderson-pages.pages.dev, fourth bullet: fine-tuning
 * computes on the packed 4-bit weights, which stay byte-identical).  The
 * gradients are the chain rule through the forward calls above; the
 * scatter-add of routed-row gradients into tokens is moe_unpermute_combine
 * with unit weights.  No weight gradient exists.
 *
 * moe_nf4_grouped_gemm_t -- out[p] = W[e(p)]^T @ G[p] for every row p in
 * expert e's segment, W[e] the NF4 weights of moe_nf4_grouped_gemm.
 *   G        F32 or F16 [G_rows >= M_total, N]   (device)
 *   packed   uint8 [E, N, K/2], absmax fp32 [E, N*K/64]  (the forward's)
 *   expert_offsets int32 [E+1] (device), monotone, offsets[E] == M_total,
 *            else MOE_DEVERR_BAD_OFFSETS and no output
 *   out      F32 or F16 [M_total, K]
 *   algo     MOE_ALGO_GEMV: CUDA-core kernel (any G dtype, K % 64 == 0);
 *            MOE_ALGO_TC: the tcgen05 kernel in its transposed form (G F16,
 *            N % 64 == 0, K % 256 == 0): each thread decodes one output
 *            column's weights down 64 rows into tensor memory, weights enter
 *            as fp16(fp16(level) * fp16(absmax)) as in the forward TC kernel;
 *            AUTO: TC when it applies and M_total >= 36 * E, else GEMV
 *   E <= 1024.  fp32 sums.  All pointers 16-byte aligned.
 */
moe_status_t moe_nf4_grouped_gemm_t(const void* G, moe_dtype_t g_dtype, int G_rows,
                                    const uint8_t* packed, const float* absmax,
                                    const int32_t* expert_offsets, int E, int N, int K,
                                    int M_total, void* out, moe_dtype_t out_dtype,
                                    moe_algo_t algo, int32_t* dev_err, void* stream);

/*
 * moe_nf4_down_backward -- the down projection's backward and the SwiGLU
 * backward in one tensor-core launch: with dh[p] = W_d[e(p)]^T @ dYp[p]
 * (the transposed grouped GEMM over the down stack [E, H, I]) and the
 * forward's gate_up pre-activations gu[p] = [g | u] (I each), s = sigmoid(g):
 *   dgu[p, i] = dh u s (1 + g (1 - s)),  dgu[p, I + i] = dh g s.
 * dh never reaches memory.  ("grouped-nf4-gemm & experts-4bit", fourth
 * bullet: the backward computes on the packed weights, fused.)
 *   dYp      F16 [G_rows >= M_total, H]   routed rows' output gradients
 *   packed   uint8 [E, H, I/2], absmax fp32 [E, H*I/64]  (the down stack)
 *   expert_offsets int32 [E+1], as above
 *   gu       fp32 [M_total, 2I]            (the forward's, gate | up)
 *   dgu      F32 or F16 [M_total, 2I]      output
 *   H % 64 == 0, I % 256 == 0, E <= 1024; other shapes MOE_ERR_UNSUPPORTED
 *   (use moe_nf4_grouped_gemm_t and moe_swiglu_backward).
 * All pointers 16-byte aligned.
 */
moe_status_t moe_nf4_down_backward(const void* dYp, int G_rows, const uint8_t* packed,
                                   const float* absmax, const int32_t* expert_offsets, int E,
                                   int H, int I, int M_total, const float* gu, void* dgu,
                                   moe_dtype_t dgu_dtype, int32_t* dev_err, void* stream);

/*
 * moe_swiglu_backward -- for gu [M, 2I] (gate | up pre-activations) and
 * dh [M, I], both of in_dtype (F32 or F16): with s = sigmoid(g),
 * dgu[m, i] = dh u s (1 + g (1 - s)) and dgu[m, I + i] = dh g s, into
 * dgu [M, 2I] of out_dtype (F32 or F16).  Pointers 16-byte aligned.
 */
moe_status_t moe_swiglu_backward(const void* gu, const void* dh, moe_dtype_t in_dtype, int M,
                                 int I, void* dgu, moe_dtype_t out_dtype, void* stream);

/*
 * moe_combine_backward -- adjoint of moe_unpermute_combine: for every routed
 * row f = t*k + j at position pos = inv_perm[f],
 *   dYp[pos, :] = topk_w[f] * dY[t, :]      (dYp [T*k, H] of dyp_dtype)
 *   dw[f]       = <dY[t, :], Yp[pos, :]>   (fp32 [T, k], fp32 sums)
 *   dY fp32 [T, H]; Yp [T*k, H] of yp_dtype (F32 or F16, the forward's);
 *   1 <= k <= 32.  An inv_perm entry out of range sets MOE_DEVERR_BAD_INDEX
 *   and that row's dw to 0.  Pointers 16-byte aligned.
 */
moe_status_t moe_combine_backward(const float* dY, const void* Yp, moe_dtype_t yp_dtype,
                                  const int32_t* inv_perm, const float* topk_w, int T, int k,
                                  int H, void* dYp, moe_dtype_t dyp_dtype, float* dw,
                                  int32_t* dev_err, void* stream);

/*
 * moe_route_backward -- gradient of the routing weights w.r.t. the logits,
 * the selection held fixed: renormalize != 0: dl[e_j] = w_j (dw_j - sum_j'
 * dw_j' w_j') and 0 elsewhere; renormalize == 0 (w = softmax probabilities):
 * dl_i = [i = e_j] dw_j w_j - p_i sum_j dw_j w_j with p = softmax(logits).
 *   logits fp32 [T, E]; topk_idx int32 [T, k] and topk_w fp32 [T, k] (the
 *   forward's outputs); dw fp32 [T, k]; dlogits fp32 [T, E].
 *   1 <= k <= min(E, 32), E <= 1024.  An expert index out of range sets
 *   MOE_DEVERR_BAD_INDEX and is skipped.  Pointers 16-byte aligned.
 */
moe_status_t moe_route_backward(const float* logits, const int32_t* topk_idx,
                                const float* topk_w, const float* dw, int T, int E, int k,
                                int renormalize, float* dlogits, int32_t* dev_err, void* stream);

/*
 * moe_lora_delta -- adds each routed row's per-expert LoRA term to an fp32
 * pre-activation in place: out[p] += scale * B[e(p)] @ (A[e(p)] @ X[p]) for
 * every row p in expert e's segment [expert_offsets[e], expert_offsets[e+1]).
 * ("Jordan Anderson", jordananderson.work, section "4-bit Mixture-of-Experts
 * fine-tuning on small GPUs": LoRA adapters per expert over the frozen 4-bit
 * base; the form W x + scale * B (A x), scale = alpha / r, is LoRA's.)  Run
 * it after moe_nf4_grouped_gemm / moe_int4_grouped_gemm with MOE_EPI_NONE and
 * F32 output, then moe_swiglu for gate_up.
 *
 *   X        fp16 [A_rows >= M_total, K]  the projection's input rows in
 *            permuted order (the GEMM's A)
 *   expert_offsets int32 [E+1] (device), monotone, offsets[0] == 0,
 *            offsets[E] == M_total, else MOE_DEVERR_BAD_OFFSETS is set and
 *            out is left unchanged
 *   E <= 1024, N >= 1, K % 8 == 0, r % 8 == 0, 8 <= r <= 64
 *   lora_A   fp16 [E, r, K]   (device, read only)
 *   lora_B   fp16 [E, N, r]   (device, read only)
 *   scale    the adapter's scale (alpha / r)
 *   out      fp32 [M_total, N] (device), read and written
 * Sums are fp32 (A X kept in fp32, not rounded to fp16).  All pointers
 * 16-byte aligned.  Shapes outside the limits return MOE_ERR_UNSUPPORTED.
 */
moe_status_t moe_lora_delta(const void* X, int A_rows, const int32_t* expert_offsets, int E,
                            int N, int K, int r, const void* lora_A, const void* lora_B,
                            float scale, int M_total, float* out, int32_t* dev_err,
                            void* stream);

/*
 * Workspace bytes moe_route_permute needs for (T, E, k).  `bytes` is a HOST
 * pointer.  Host-only, no CUDA call.
 */
moe_status_t moe_route_permute_workspace_size(int T, int E, int k,
                                              size_t* bytes);

/*
 * moe_route_permute -- top-k softmax routing and the token->expert
 * permutation.  (The router of "grouped-nf4-gemm & experts-4bit", second
 * bullet; the per-expert row segments one grouped launch needs, first
 * bullet.)
 *
 *   logits         fp32  [T, E]   router logits (device)
 *   T >= 0; 1 <= E <= 1024; 1 <= k <= min(E, 32)
 *   renormalize    1: weights = softmax over the k chosen logits;
 *                  0: weights = softmax over all E logits, taken at the k
 *   topk_idx       int32 [T, k]   chosen experts, descending logit, equal
 *                                 logits -> lower expert index first
 *   topk_w         fp32  [T, k]   routing weights
 *   expert_offsets int32 [E+1]    segment starts; offsets[E] == T*k
 *   sorted_rows    int32 [T*k]    flat id t*k+j at each permuted position,
 *                                 stable: by expert, then by flat id
 *   inv_perm       int32 [T*k]    permuted position of each flat id
 *   workspace      device scratch of moe_route_permute_workspace_size bytes
 * Indices, offsets and the permutation are deterministic and bit-exact;
 * the weights are fp32 (expf, fixed reduction order).  Logits must be
 * finite.  All pointers 16-byte aligned.
 */
moe_status_t moe_route_permute(const float* logits, int T, int E, int k,
                               int renormalize, int32_t* topk_idx,
                               float* topk_w, int32_t* expert_offsets,
                               int32_t* sorted_rows, int32_t* inv_perm,
                               void* workspace, size_t workspace_bytes,
                               void* stream);

/*
 * moe_route_permute_noalloc -- moe_route_permute without a workspace argument.
 * (The pages have no counterpart: this entry point exists for callers of this
 * library that cannot allocate device memory where they route, e.g. a host
 * framework that owns all device memory through its own allocator, or a
 * latency-critical loop in which cudaMalloc, which may synchronize the
 * device, is not acceptable.)
 *
 * Arguments, outputs and results are those of moe_route_permute.  The scratch
 * lives in a fixed array of MOE_ROUTE_NOALLOC_SCRATCH_BYTES bytes of device
 * memory inside the library; every GPU that loads the library holds it until
 * the process exits.  The call allocates nothing and frees nothing.
 * - Size limit: moe_route_permute_workspace_size(T, E, k) must not exceed
 *   MOE_ROUTE_NOALLOC_SCRATCH_BYTES (T*k up to about 200,000 routed rows at
 *   E = 128); larger problems return MOE_ERR_WORKSPACE and enqueue nothing.
 * - Set-up: the first call in each CUDA context (normally a device's
 *   primary context) looks up the array's device address there
 *   (cudaGetSymbolAddress) and caches it for that context; make that first
 *   call before any stream capture on the device.
 * - Sharing: all calls on a device use the same array, which keeps the last
 *   call's contents (nothing in it needs to start at zero).  Calls whose
 *   kernels overlap on the GPU -- on different streams, or from different
 *   host threads -- race on the array and give wrong results; serialize them.
 */
#define MOE_ROUTE_NOALLOC_SCRATCH_BYTES (1u << 20)
moe_status_t moe_route_permute_noalloc(const float* logits, int T, int E, int k,
                                       int renormalize, int32_t* topk_idx,
                                       float* topk_w, int32_t* expert_offsets,
                                       int32_t* sorted_rows, int32_t* inv_perm,
                                       void* stream);

/*
 * moe_nf4_grouped_gemm -- one launch over all experts:
 *   out[p, :] = W[e(p)] . A[r(p), :]   for p in [0, M_total)
 * where e(p) is the expert whose segment [offsets[e], offsets[e+1]) holds p
 * and r(p) = gather[p] / k when `gather` is given (the routed token of the
 * permuted row), else p.  The NF4 weights are decoded in registers.
 * ("grouped-nf4-gemm & experts-4bit", first bullet: one launch for all active
 * experts, codebook decoded inside the GEMM, no dequantize-to-bf16 round
 * trip.)
 *
 *   A        [A_rows, K] BF16 or F16 activations; with `gather` A holds the
 *            T tokens (A_rows = T), without it one row per position
 *            (A_rows >= M_total, checked on the host)
 *   gather   int32 [M_total] or NULL; k = the routing top-k (used with
 *            gather only).  A gathered id f must satisfy 0 <= f < M_total
 *            and f / k < A_rows, else MOE_DEVERR_BAD_INDEX is set and the
 *            row is computed as zeros
 *   packed   uint8 [E, N, K/2], absmax fp32 [E, N*K/64]
 *   expert_offsets int32 [E+1], monotone, offsets[E] == M_total (checked on
 *            the device: violation -> MOE_DEVERR_BAD_OFFSETS, no output)
 *   N % 64 == 0 (for SWIGLU N = 2I); K % 64 == 0
 *   epilogue NONE:   out [M_total, N]
 *            SWIGLU: out [M_total, N/2] = silu(g) * u with g the first N/2
 *                    outputs (gate rows) and u the last N/2 (up rows)
 *   out_dtype F32, BF16 or F16 (rounded once from the fp32 accumulator)
 *   algo     MOE_ALGO_AUTO / _GEMV / _TC
 * Accumulation is fp32; activations enter the tensor cores as fp16.
 * GEMV kernel: weights enter as the fp16 rounding of each level, the fp32
 * absmax multiplies each 64-element block's fp32 partial sum.
 * TC kernel (tcgen05): weights enter as fp16(fp16(level) * fp16(absmax));
 * it needs gather == NULL and F16 A (rows already permuted, e.g. by
 * moe_permute_rows), N % 128 == 0, absmax < 65504.  AUTO uses it when those
 * hold and M_total >= 36 * E.  A call WITH `gather` therefore never reaches
 * the tensor cores: it always runs the general GEMV kernel (MOE_ALGO_TC then
 * returns MOE_ERR_UNSUPPORTED); prefill-sized callers permute first.
 * An absmax that is not 0 and lies outside [2^-14, 65504) -- where
 * fp16(absmax) is subnormal or not finite -- sets MOE_DEVERR_RANGE in the
 * TC kernel (the result then carries fp16 underflow error).
 * All pointers 16-byte aligned.
 */
moe_status_t moe_nf4_grouped_gemm(const void* A, moe_dtype_t a_dtype,
                                  int A_rows, const int32_t* gather, int k,
                                  const uint8_t* packed, const float* absmax,
                                  const int32_t* expert_offsets, int E, int N,
                                  int K, int M_total, moe_epilogue_t epilogue,
                                  void* out, moe_dtype_t out_dtype,
                                  moe_algo_t algo, int32_t* dev_err,
                                  void* stream);

/*
 * moe_permute_rows -- gathers the routed activation rows into permuted
 * order, converted to fp16: Xp[p, :] = fp16(X[sorted_rows[p] / k, :]) for
 * p < M_total.  This is the activation side of the permutation (the
 * permuted rows one grouped launch reads as contiguous per-expert
 * segments, "grouped-nf4-gemm & experts-4bit", first bullet); the decode
 * and tensor-core grouped GEMMs read their activations this way, through
 * TMA.
 *   X   [T, K] BF16 or F16; sorted_rows int32 [M_total]; Xp fp16 [M_total, K]
 *   K % 8 == 0; ids with f < 0, f >= M_total or f / k >= T give zero rows
 *   and MOE_DEVERR_BAD_INDEX.  Pointers 16-byte aligned.
 */
moe_status_t moe_permute_rows(const void* X, moe_dtype_t x_dtype, int T, int K,
                              const int32_t* sorted_rows, int k, int M_total,
                              void* Xp, int32_t* dev_err, void* stream);

/*
 * moe_swiglu -- standalone h[m, i] = silu(gu[m, i]) * gu[m, I + i],
 * silu(g) = g / (1 + exp(-g)), for gu [M, 2I] (F32, BF16 or F16) into
 * h [M, I] of h_dtype.  (The pages name the experts' matmuls but not their
 * activation; the SiLU(gate) * up step between the two grouped projections
 * is fixed by the problem statement this library implements.)  The fused
 * path never calls this -- the gate_up GEMM applies it in its epilogue; it
 * exists for callers that keep gate_up outputs (e.g. to add a LoRA term
 * first).  I % 4 == 0, pointers 16-byte aligned.
 */
moe_status_t moe_swiglu(const void* gu, moe_dtype_t gu_dtype, int M, int I,
                        void* h, moe_dtype_t h_dtype, void* stream);

/*
 * moe_unpermute_combine -- Y[t, :] = sum_{j<k} topk_w[t, j] *
 * Yp[inv_perm[t*k + j], :], summed in j order in fp32.  (The pages print no
 * formula for it; the routing-weighted scatter-combine that closes the layer
 * is fixed by the problem statement this library implements, and it is the
 * inverse of the permutation of moe_route_permute.)
 *   Yp [T*k, H] of yp_dtype (F32, BF16, F16), Y [T, H] of y_dtype.
 *   1 <= k <= 32, H % 4 == 0, pointers 16-byte aligned.
 */
moe_status_t moe_unpermute_combine(const void* Yp, moe_dtype_t yp_dtype,
                                   const int32_t* inv_perm,
                                   const float* topk_w, int T, int k, int H,
                                   void* Y, moe_dtype_t y_dtype,
                                   void* stream);

/*
 * Whole layer in one call (route -> permute -> gate_up+SwiGLU -> down ->
 * combine), each step the entry point above, all on `stream`.  The two
 * grouped GEMMs run chained (each requests its first weights while the
 * kernel before it finishes).
 *   X bf16 [T, H]; logits fp32 [T, E]; gate_up stack [E, 2I, H];
 *   down stack [E, H, I]; Y fp32 [T, H].
 *   workspace: moe_layer_workspace_size bytes; it holds the routing outputs
 *   and the fp16 intermediates [T*k, H] (permuted X), [T*k, I] and
 *   [T*k, H].
 */
moe_status_t moe_layer_workspace_size(int T, int E, int k, int H, int I,
                                      size_t* bytes);
moe_status_t moe_layer_forward(const void* X, const float* logits, int T,
                               int E, int k, int renormalize, int H, int I,
                               const uint8_t* packed_gu,
                               const float* absmax_gu,
                               const uint8_t* packed_d, const float* absmax_d,
                               float* Y, void* workspace,
                               size_t workspace_bytes, int32_t* dev_err,
                               void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_NF4_H */
