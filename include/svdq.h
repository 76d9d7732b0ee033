/*
 * svdq.h -- C ABI of the B200 (sm_100a) SVDQuant W4A4 + low-rank linear layer.
 *
 * The layer is the one of "SVDQuant: Absorbing Outliers by Low-Rank
 * Components for 4-Bit Diffusion Models" (arXiv 2411.05007), Sec. 4.2, Eq. 5:
 *
 *     Y = X_hat L1 L2 + Q(X_hat) Q(R) + bias,     X_hat = X diag(lambda)^-1,
 *
 * where lambda smooths each input channel, L1 (K x r) and L2 (r x N) are the
 * 16-bit rank-r factors of the smoothed weight W_hat = diag(lambda) W from its
 * truncated SVD, R = W_hat - L1 L2 is the residual, and Q is the symmetric
 * per-group 4-bit quantizer of Sec. 3.  Two 4-bit formats are supported:
 *   SVDQ_NVFP4: E2M1 codes with one E4M3 scale per 16 values along K;
 *   SVDQ_INT4 : signed 4-bit integers in [-7, 7] with one fp16 scale per 64
 *               values along K (Sec. 5.1);
 *   SVDQ_FP4G32: E2M1 codes with one E4M3 scale per 32 values along K (the
 *               paper's FP4 setting of Sec. 5.1: groups of 32, an FP8 scale).
 *               It runs on the NVFP4 kernels with each scale stored twice.
 *   SVDQ_W8A8 : the 8-bit setting of Sec. 5.1: int8 codes in [-127, 127],
 *               one fp32 scale per token for the activations (computed on the
 *               fly over all of K) and one per output channel for the
 *               weights; the integer dot product is exact and scaled once.
 *               The paper pairs it with rank 16.
 *
 * Conventions for every call:
 *   - "device" pointers are CUDA global-memory pointers on the current device;
 *     "host" pointers are ordinary CPU memory.  The caller owns every pointer
 *     it passes; the library owns the memory behind an svdq_weights handle.
 *   - bf16 tensors are raw IEEE bfloat16 (2 bytes), row-major and contiguous.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  The hot
 *     calls (svdq_quantize_act, svdq_linear, svdq_forward) are asynchronous on
 *     it, never allocate and never synchronize.  Preparation, LoRA appending
 *     and the export calls may allocate and synchronize.
 *   - Every call returns an svdq_status; on failure nothing has been launched
 *     unless the status is SVDQ_ERR_CUDA.
 *
 * Shape rules: K % 64 == 0, N % 16 == 0, M >= 0 (M == 0 is a no-op),
 * 0 <= rank (+ LoRA rank) <= 256 and rank <= min(K, N).  Device pointers to
 * X, Y and the workspace must be 16-byte aligned (cudaMalloc gives 256).
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SVDQ_API __attribute__((visibility("default")))
#else
#define SVDQ_API
#endif

typedef enum {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,       /* null pointer, bad enum, misaligned pointer */
  SVDQ_ERR_UNSUPPORTED_SHAPE = 2, /* violates the shape rules above */
  SVDQ_ERR_ALLOC = 3,             /* a preparation-time cudaMalloc failed */
  SVDQ_ERR_CUDA = 4,              /* a CUDA runtime / driver call failed */
  SVDQ_ERR_TIMEOUT = 5,           /* a bounded device wait ran out (svdq_get_error) */
  SVDQ_ERR_LIBRARY = 6            /* cuSOLVER / cuBLAS failed during preparation */
} svdq_status;

typedef enum { SVDQ_NVFP4 = 0, SVDQ_INT4 = 1, SVDQ_FP4G32 = 2, SVDQ_W8A8 = 3 } svdq_format;

/* Opaque prepared layer: 4-bit residual codes and scales, the bf16 low-rank
 * factors, 1/lambda and the bias, all in device memory owned by the handle. */
typedef struct svdq_weights svdq_weights;

/* Inputs of svdq_prepare_weights (all device pointers). */
/* Preparation flags.
 * SVDQ_WEIGHT_POW2_PRESCALE (FP4 formats; ignored by INT4 and W8A8): quantize
 *   the residual as R * 2^e, e the largest integer with 2^e * max|R| / 6 <= 448,
 *   so that small residuals keep normal E4M3 group scales (the E4M3 range ends
 *   in subnormals near 2^-9, and a weight whose group maxima sit near 10^-3
 *   would lose its scales there); the GEMM multiplies its group sum by 2^-e
 *   (exact) before the low-rank branch and the bias are added.  The paper has
 *   no global scale for its 4-bit groups; off by default.  The exponent is
 *   reported by svdq_weights_scale_exponent; the exported codes and scales are
 *   those of R * 2^e. */
#define SVDQ_WEIGHT_POW2_PRESCALE 1u

typedef struct {
  int fmt;                 /* svdq_format */
  int K, N;                /* W is K x N: input channels x output channels */
  int rank;                /* r of the SVD branch, 0 = plain W4A4 */
  const void* W;           /* bf16 K x N */
  const float* x_absmax;   /* K calibration maxima max|X_j|, or NULL (lambda = 1) */
  const void* bias;        /* bf16 N, or NULL */
  const void* lora_A;      /* bf16 K x lora_rank, or NULL */
  const void* lora_B;      /* bf16 lora_rank x N, or NULL */
  int lora_rank;           /* 0 = no LoRA */
  int refine_iters;        /* iterative updates of the low-rank branch (Sec. 4.2), 0 = none */
  unsigned flags;          /* SVDQ_WEIGHT_POW2_PRESCALE or 0 */
} svdq_prepare_desc;

/* Inputs of svdq_load_weights: an already decomposed layer (device pointers). */
typedef struct {
  int fmt, K, N, rank;
  const float* inv_lambda; /* K values of 1/lambda, or NULL (all ones) */
  const float* lambda;     /* K values of lambda (used by svdq_append_lora), or NULL = 1/inv_lambda */
  const void* L1;          /* bf16 K x rank (ignored if rank == 0) */
  const void* L2;          /* bf16 rank x N (ignored if rank == 0) */
  const float* R;          /* fp32 K x N residual, quantized here */
  const void* bias;        /* bf16 N, or NULL */
  unsigned flags;          /* SVDQ_WEIGHT_POW2_PRESCALE or 0 */
} svdq_parts_desc;

/* Calibration statistic for the smoothing factor (Sec. 4.2):
 * absmax[k] = max(absmax[k], max_m |X[m, k]|) if accumulate != 0, else
 * absmax[k] = max_m |X[m, k]|.  X: device bf16 M x K; absmax: device float K.
 * Asynchronous on `stream`. */
SVDQ_API int svdq_calib_absmax(const void* X, int M, int K, float* absmax, int accumulate,
                               void* stream);

/* Offline preparation (Sec. 4.2 and Sec. 5.2): lambda_j = sqrt(max|X_j| /
 * max|W_j|) (fp64, rounded to fp32); W_hat = diag(lambda) W; the optimal
 * rank-r factors from the eigen-decomposition of the fp64 Gram matrix of
 * W_hat (cuSOLVER), rounded to bf16; R = W_hat - L1 L2; Q(R); optional LoRA
 * folded into the branch without requantizing R.  With refine_iters = T > 0
 * the branch is updated T times (Sec. 4.2, last paragraph): the rank-r factors
 * of E = W_hat - deq(Q(R)) replace L1, L2, R = W_hat - L1 L2 is requantized,
 * and the iterate (the SVD start included) with the smallest
 * ||W_hat - L1 L2 - deq(Q(R))||_F is kept (before any LoRA is folded in).
 * Allocates device memory (SVDQ_ERR_ALLOC) and synchronizes `stream`.
 * *out receives a new handle. */
SVDQ_API int svdq_prepare_weights(const svdq_prepare_desc* desc, void* stream,
                                  svdq_weights** out);

/* Build a handle from given factors (e.g. a layer prepared offline elsewhere):
 * copies 1/lambda, lambda, L1, L2 and the bias, and quantizes R on the device
 * with the same quantizer as svdq_prepare_weights.  Synchronizes `stream`. */
SVDQ_API int svdq_load_weights(const svdq_parts_desc* desc, void* stream, svdq_weights** out);

/* Fold a LoRA (A: bf16 K x lora_rank, B: bf16 lora_rank x N, device) into the
 * low-rank branch (Sec. 5.2): L1 <- [L1 | bf16(diag(lambda) A)], L2 <- [L2 ; B].
 * The 4-bit residual codes are not touched.  Synchronizes `stream`. */
SVDQ_API int svdq_append_lora(svdq_weights* w, const void* lora_A, const void* lora_B,
                              int lora_rank, void* stream);

/* Weight error ||W_hat - L1 L2 - deq(Q(R))||_F of the SVD start and of the
 * kept iterate of svdq_prepare_weights' refinement (both -1 without it). */
SVDQ_API int svdq_weights_refine_error(const svdq_weights* w, double* initial, double* kept);

/* The weight prescale exponent e of a handle (0 without SVDQ_WEIGHT_POW2_PRESCALE). */
SVDQ_API int svdq_weights_scale_exponent(const svdq_weights* w, int* exponent);

/* Shape of a handle; any output pointer may be NULL. */
SVDQ_API int svdq_weights_info(const svdq_weights* w, int* fmt, int* K, int* N, int* rank,
                               int* rank_padded);

/* Bytes of the activation workspace svdq_quantize_act fills for M tokens
 * (codes, scales and X_hat L1).  The caller allocates it (device, 256-byte
 * aligned) and may reuse it across calls with the same or smaller M. */
SVDQ_API int svdq_act_workspace_bytes(const svdq_weights* w, int M, size_t* bytes);

/* Fused activation kernel (Sec. 4.3, "quantize + down-projection"): one pass
 * over X (device bf16 M x K) writes Q(X diag(lambda)^-1) codes and scales and
 * X_hat L1 = X (diag(lambda)^-1 L1) (fp32 precision, as a bf16 hi/lo pair)
 * into `workspace`.  Asynchronous on `stream`. */
SVDQ_API int svdq_quantize_act(const svdq_weights* w, const void* X, int M, void* workspace,
                               void* stream);

/* Fused 4-bit GEMM + up-projection + bias (Sec. 4.3): Y (device bf16 M x N) =
 * Q(X_hat) Q(R) + (X_hat L1) L2 + bias, from a workspace that
 * svdq_quantize_act filled for the same M.  Asynchronous on `stream`. */
SVDQ_API int svdq_linear(const svdq_weights* w, const void* workspace, int M, void* Y,
                         void* stream);

/* svdq_quantize_act followed by svdq_linear. */
SVDQ_API int svdq_forward(const svdq_weights* w, const void* X, int M, void* Y, void* workspace,
                          void* stream);

/* Fixed size of the device workspace array behind svdq_forward_noalloc. */
#define SVDQ_NOALLOC_WORKSPACE_BYTES (16u << 20)

/* svdq_forward without a caller workspace and without any allocation.  The
 * paper has no counterpart: this is for callers that cannot call cudaMalloc,
 * e.g. a plugin whose host framework owns all device memory, or a serving
 * loop that must not pay cudaMalloc's implicit device synchronization.  The
 * activation workspace lives in a fixed __device__ array of
 * SVDQ_NOALLOC_WORKSPACE_BYTES (16 MiB) that every GPU loading the library
 * keeps until exit.  M is limited to what fits: svdq_act_workspace_bytes(w, M)
 * must be <= SVDQ_NOALLOC_WORKSPACE_BYTES (for K = 3072, rank 32, NVFP4: about
 * 9000 tokens), else SVDQ_ERR_UNSUPPORTED_SHAPE and nothing is launched.
 * The first call on a device looks up the array's address (do it before any
 * stream capture).  All calls on a device share the one array: calls that
 * overlap on the GPU (other streams, other threads) race and must be
 * serialized by the caller.  X, Y, stream: as for svdq_forward. */
SVDQ_API int svdq_forward_noalloc(const svdq_weights* w, const void* X, int M, void* Y, void* stream);

/* Debug export of a filled workspace in plain layouts (host outputs, any may
 * be NULL; synchronizes the device):
 *   codes  M x K/2 bytes, element 2i in the low nibble (INT4: two's complement);
 *          W8A8: M x K int8;
 *   scales M x K/16 E4M3 bytes (NVFP4), M x K/32 E4M3 bytes (FP4 g32),
 *          M x K/64 fp16 (INT4) or M fp32 (W8A8);
 *   xl1    M x rank fp32 (X_hat L1 at fp32 precision; stored as a bf16 pair). */
SVDQ_API int svdq_export_act(const svdq_weights* w, const void* workspace, int M,
                             uint8_t* codes, void* scales, void* xl1);

/* Debug export of a handle in plain layouts (host outputs, any may be NULL):
 *   codes N x K/2 (per output column, along K; W8A8: N x K int8), scales
 *   N x K/16, N x K/32, N x K/64 (as for svdq_export_act) or N fp32 (W8A8),
 *   L1 K x rank bf16, L2 rank x N bf16, inv_lambda K floats, lambda K floats. */
SVDQ_API int svdq_export_weights(const svdq_weights* w, uint8_t* codes, void* scales, void* L1,
                                 void* L2, float* inv_lambda, float* lambda);

/* Sticky device error word of the current device: bit 0 = a bounded wait ran
 * out in the activation kernel, bit 1 = in a GEMM kernel.  Reading clears it.
 * Returns the word (>= 0) or -SVDQ_ERR_CUDA.  Synchronizes the device. */
SVDQ_API int svdq_get_error(void);

/* Clock-cycle budget of every bounded device wait of the hot pipelines
 * (default 2^31, about one second; the environment variable
 * SVDQ_WAIT_BUDGET_CYCLES also sets it).  A wait that runs out sets the error
 * word above and stops its CTA's pipeline; the waits with which a CTA then
 * drains what it already issued (copies landing, MMAs retiring, before shared
 * memory and TMEM are released) get max(budget, 2^33) cycles, since issued
 * work always finishes.  cycles <= 0: SVDQ_ERR_INVALID_ARG. */
SVDQ_API int svdq_set_wait_budget(long long cycles);

/* Launch shape of the activation kernel for every later svdq_quantize_act
 * (process-wide; a tuning and testing aid).  S = stacked 64-wide K sub-tiles
 * per pipeline stage (rows per CTA cluster = 128 / S), C = CTAs per cluster,
 * each on its own K range, whose partial X_hat L1 sums meet in distributed
 * shared memory.  S, C in {1, 2, 4, 8}; 0, 0 restores the automatic choice
 * (a cost model over the SM count and the resident clusters of each size).
 * A forced shape the layer cannot use (S above 256 / rank_padded, C above
 * 128 / S or above the number of stages, no resident cluster of C CTAs)
 * falls back to the automatic choice for that call.  The results do not
 * depend on the shape beyond the summation order of X_hat L1 (fp32).
 * SVDQ_ERR_INVALID_ARG for other values. */
SVDQ_API int svdq_set_quant_split(int S, int C);

/* Tile order of the GEMM for every later svdq_linear (process-wide; a tuning
 * and testing aid).  The persistent GEMM walks its output tiles (128 rows
 * per row block; 256 or 192 weight columns per column block) in groups of
 * `group_m` row blocks: all of a group's tiles, row block
 * fastest, before the next group.  Small groups keep fewer activation row
 * blocks and more weight column blocks in flight at once.  group_m above the
 * number of row blocks is clamped to it (one group: the whole of M for each
 * weight column block); 0 restores the automatic choice.  The result does not
 * depend on the order.  SVDQ_ERR_INVALID_ARG for group_m < 0. */
SVDQ_API int svdq_set_gemm_raster(int group_m);

/* GEMM kernel of the FP4 formats for every later svdq_linear (process-wide; a
 * tuning and testing aid): 1 = one CTA per 128 x 256 output tile, 2 = a pair of
 * CTAs (a cluster of two) per 256 x 256 tile, each CTA staging its own 128 rows
 * of the activations and half of the weight columns for tcgen05 MMAs that span
 * both; when the tiles left after the last full round of the pairs are at most
 * half as many as the pairs, each of them is computed as two 256 x 128 halves
 * on two pairs, 3 = a pair of CTAs per 256 x 192 tile with two accumulators in
 * TMEM (the next tile's MMAs do not wait for the epilogue), 4 = as 2 with whole
 * tiles only; 0 restores the automatic choice (3 for K <= 4096, else 2).  All
 * give the same Y bit for bit (the same products summed in the same order).
 * The INT4 and W8A8 formats have one kernel each and ignore it.  With kinds 2
 * to 4 the raster group of svdq_set_gemm_raster counts 128-row blocks and is
 * rounded up to pairs.  SVDQ_ERR_INVALID_ARG for other values. */
SVDQ_API int svdq_set_gemm_kernel(int kind);

SVDQ_API const char* svdq_status_string(int status);

/* Measurement helper, not a step of the layer: every SM of the current device
 * issues `steps` 256-wide K steps of the GEMM's own tensor-core instruction
 * (NVFP4: 4 x tcgen05.mma kind::mxf4nvf4 M=128 N=256 K=64; INT4: 4 x kind::i8
 * M=128 N=256 K=32) back to back from shared memory, with no global-memory
 * traffic.  Timing it with events on `stream` gives the tensor-core ceiling:
 *   FLOP = SMs * steps * 4 * 2 * 128 * 256 * (64 for NVFP4, 32 for INT4).
 * Asynchronous; returns SVDQ_ERR_INVALID_ARG for a bad format or steps < 1. */
SVDQ_API int svdq_tensor_peak(int fmt, long long steps, void* stream);

SVDQ_API void svdq_weights_destroy(svdq_weights* w);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H_ */
