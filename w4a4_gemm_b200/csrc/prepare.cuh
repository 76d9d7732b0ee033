// prepare.cuh -- one-time weight preparation kernels (not on the timed path).
//
// SVDQuant Sec. 4.2: smoothing W_hat = diag(lambda) W, the optimal rank-r
// factors of W_hat from its SVD (Eckart-Young-Mirsky), the residual
// R = W_hat - L1 L2 and its 4-bit per-group quantization; Sec. 5.2: a LoRA
// joins the low-rank branch (L1' = [L1 | diag(lambda) A], L2' = [L2 ; B])
// with R left as it is.
#pragma once

#include "svdq_formats.cuh"
#include "svdq_ptx.cuh"

namespace svdq {

// ------------------------------------------------------------ calibration ---
// absmax[k] = max(absmax[k], max_m |X[m, k]|): one thread per column pair,
// rows split across blockIdx.y; non-negative floats order like their bits.
__global__ void calib_absmax_kernel(const __nv_bfloat16* __restrict__ X, int M, int K,
                                    float* __restrict__ absmax) {
  const int k2 = blockIdx.x * blockDim.x + threadIdx.x;   // column pair
  if (2 * k2 >= K) return;
  const int rows_per = (M + gridDim.y - 1) / gridDim.y;
  const int r0 = blockIdx.y * rows_per, r1 = min(M, r0 + rows_per);
  float a0 = 0.f, a1 = 0.f;
  const uint32_t* x = reinterpret_cast<const uint32_t*>(X);
  for (int m = r0; m < r1; ++m) {
    const uint32_t w = __ldg(x + (static_cast<size_t>(m) * K) / 2 + k2);
    a0 = fmaxf(a0, fabsf(bf16_lo(w)));
    a1 = fmaxf(a1, fabsf(bf16_hi(w)));
  }
  atomicMax(reinterpret_cast<unsigned int*>(absmax) + 2 * k2, __float_as_uint(a0));
  atomicMax(reinterpret_cast<unsigned int*>(absmax) + 2 * k2 + 1, __float_as_uint(a1));
}

// wmax[k] = max_n |W[k, n]| (one block per input channel k).
__global__ void row_absmax_kernel(const __nv_bfloat16* __restrict__ W, int K, int N,
                                  float* __restrict__ wmax) {
  const int k = blockIdx.x;
  float a = 0.f;
  for (int n = threadIdx.x; n < N; n += blockDim.x)
    a = fmaxf(a, fabsf(__bfloat162float(W[static_cast<size_t>(k) * N + n])));
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  __shared__ float red[32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x < 32) {
    a = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (threadIdx.x == 0) wmax[k] = a;
  }
}

// lambda_k = sqrt(max|X_k| / max|W_k|) in fp64, rounded to fp32 (1 where either
// maximum is 0 or no calibration is given); inv_lambda = fp32 1 / lambda.
__global__ void smoothing_kernel(const float* __restrict__ xmax, const float* __restrict__ wmax,
                                 int K, float* __restrict__ lam, float* __restrict__ inv) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  float l = 1.0f;
  if (xmax != nullptr) {
    const double xm = xmax[k], wm = wmax[k];
    if (xm > 0.0 && wm > 0.0) l = static_cast<float>(sqrt(xm / wm));
  }
  lam[k] = l;
  inv[k] = __fdiv_rn(1.0f, l);
}

// W_hat[k, n] = lambda_k * W[k, n] in fp64 (exact).
__global__ void smooth_weight_kernel(const __nv_bfloat16* __restrict__ W,
                                     const float* __restrict__ lam, int K, int N,
                                     double* __restrict__ What) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<size_t>(K) * N) return;
  const int k = static_cast<int>(i / N);
  What[i] = static_cast<double>(lam[k]) * static_cast<double>(__bfloat162float(W[i]));
}

// Nearest bf16 of a finite double (ties to even), from the bit fields: keep 8
// significant bits of the 53, rounding the dropped 45 to nearest even.
__device__ __forceinline__ __nv_bfloat16 bf16_from_f64(double x) {
  if (x == 0.0) return __float2bfloat16_rn(static_cast<float>(x));
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(x));
  const unsigned long long sign = b >> 63;
  int e = static_cast<int>((b >> 52) & 0x7FF) - 1023;
  unsigned long long mant = (b & ((1ull << 52) - 1)) | (1ull << 52);
  if (e < -126) {
    // below the normal bf16 range: fall back to the float path (values that
    // small never occur in these factors)
    return __float2bfloat16_rn(static_cast<float>(x));
  }
  unsigned long long kept = mant >> 45;
  const unsigned long long rem = mant & ((1ull << 45) - 1), half = 1ull << 44;
  if (rem > half || (rem == half && (kept & 1ull))) ++kept;
  if (kept == (1ull << 8)) {
    kept >>= 1;
    ++e;
  }
  const uint32_t fbits = static_cast<uint32_t>(sign << 31) |
                         (static_cast<uint32_t>(e + 127) << 23) |
                         (static_cast<uint32_t>(kept & 0x7Full) << 16);
  return __float2bfloat16_rn(__uint_as_float(fbits));   // exact: already 8 significant bits
}

// Low-rank factors from the eigenvectors of the Gram matrix (column-major,
// ascending eigenvalues), written straight into the kernel layouts
//   L1t[j][k] = bf16(L1[k, j])  (r_pad x K),   L2t[n][j] = bf16(L2[j, n])  (N x r_pad).
// gram_left: G = W_hat W_hat^T (K x K), eigenvectors u_j; L1 = u_j sigma_j,
//            L2 = u_j^T W_hat / sigma_j.
// else     : G = W_hat^T W_hat (N x N), eigenvectors v_j; L2 = v_j^T, L1 = W_hat v_j.
__global__ void lowrank_l1_kernel(const double* __restrict__ evec, const double* __restrict__ eval,
                                  const double* __restrict__ What, int K, int N, int r, int r_pad,
                                  int gram_left, __nv_bfloat16* __restrict__ l1t,
                                  double* __restrict__ l1_f64) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  const int j = blockIdx.y;
  if (k >= K) return;
  double v = 0.0;
  if (j < r) {
    if (gram_left) {
      const int col = K - 1 - j;
      v = evec[static_cast<size_t>(col) * K + k] * sqrt(fmax(eval[col], 0.0));
    } else {
      const int col = N - 1 - j;
      const double* vj = evec + static_cast<size_t>(col) * N;
      const double* wr = What + static_cast<size_t>(k) * N;
      for (int n = 0; n < N; ++n) v += wr[n] * vj[n];
    }
  }
  l1t[static_cast<size_t>(j) * K + k] = j < r ? bf16_from_f64(v) : __float2bfloat16_rn(0.f);
  if (l1_f64 != nullptr && j < r) l1_f64[static_cast<size_t>(k) * r + j] = v;
}

__global__ void lowrank_l2_kernel(const double* __restrict__ evec, const double* __restrict__ eval,
                                  const double* __restrict__ What, int K, int N, int r, int r_pad,
                                  int gram_left, __nv_bfloat16* __restrict__ l2t) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int j = blockIdx.y;
  if (n >= N) return;
  double v = 0.0;
  if (j < r) {
    if (gram_left) {
      const int col = K - 1 - j;
      const double sigma = sqrt(fmax(eval[col], 0.0));
      const double* uj = evec + static_cast<size_t>(col) * K;
      for (int k = 0; k < K; ++k) v += uj[k] * What[static_cast<size_t>(k) * N + n];
      v = sigma > 0.0 ? v / sigma : 0.0;
    } else {
      v = evec[static_cast<size_t>(N - 1 - j) * N + n];
    }
  }
  l2t[static_cast<size_t>(n) * r_pad + j] = j < r ? bf16_from_f64(v) : __float2bfloat16_rn(0.f);
}

// Re-layout caller-given factors: L1 (K x r, bf16 row-major) -> L1t (r_pad x K);
// L2 (r x N) -> L2t (N x r_pad); padding is zero.  `col0` places them at
// branch columns [col0, col0 + r) (used when a LoRA is appended).
__global__ void layout_l1_kernel(const __nv_bfloat16* __restrict__ L1, int K, int r, int col0,
                                 __nv_bfloat16* __restrict__ l1t) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  const int j = blockIdx.y;
  if (k >= K || j >= r) return;
  l1t[static_cast<size_t>(col0 + j) * K + k] = L1[static_cast<size_t>(k) * r + j];
}

__global__ void layout_l2_kernel(const __nv_bfloat16* __restrict__ L2, int N, int r, int col0,
                                 int r_pad, __nv_bfloat16* __restrict__ l2t) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int j = blockIdx.y;
  if (n >= N || j >= r) return;
  l2t[static_cast<size_t>(n) * r_pad + col0 + j] = L2[static_cast<size_t>(j) * N + n];
}

// Copy branch columns [0, r_old) of the old layouts into wider ones.
__global__ void widen_l1_kernel(const __nv_bfloat16* __restrict__ old_t, int K, int r_old,
                                __nv_bfloat16* __restrict__ new_t) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < static_cast<size_t>(K) * r_old) new_t[i] = old_t[i];
}

__global__ void widen_l2_kernel(const __nv_bfloat16* __restrict__ old_t, int N, int r_old,
                                int r_pad_old, int r_pad_new, __nv_bfloat16* __restrict__ new_t) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  for (int j = 0; j < r_old; ++j)
    new_t[static_cast<size_t>(n) * r_pad_new + j] = old_t[static_cast<size_t>(n) * r_pad_old + j];
}

// LoRA A joins L1 as bf16(lambda_k * A[k, j]) (X A = X_hat diag(lambda) A).
__global__ void lora_l1_kernel(const __nv_bfloat16* __restrict__ A, const float* __restrict__ lam,
                               int K, int rl, int col0, __nv_bfloat16* __restrict__ l1t) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  const int j = blockIdx.y;
  if (k >= K || j >= rl) return;
  const double v = static_cast<double>(lam[k]) *
                   static_cast<double>(__bfloat162float(A[static_cast<size_t>(k) * rl + j]));
  l1t[static_cast<size_t>(col0 + j) * K + k] = bf16_from_f64(v);
}

// The smoothing folded into the down-projection factor, carried as a pair of
// bf16 terms so that it keeps 16 bits more than one bf16 rounding would:
//   p = inv_lambda[k] * l1t[j][k]           (exact in fp64: 24 x 8 bits)
//   l1st[j][k]         = hi = bf16(p)
//   l1st[r_pad + j][k] = lo = bf16(p - hi)  (p - hi exact in fp64)
// |hi + lo - p| <= 2^-8 |p - hi| <= 2^-16 |p|.  The activation kernel computes
// X hi + X lo = X (diag(lambda)^-1 L1) = X_hat L1 (SVDQuant Sec. 4.2) with the
// X tile as loaded; every product of two bf16 values is exact in fp32.
__global__ void fold_l1_kernel(const __nv_bfloat16* __restrict__ l1t, const float* __restrict__ inv,
                               int K, int r, int r_pad, __nv_bfloat16* __restrict__ l1st) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  const int j = blockIdx.y;
  if (k >= K || j >= r) return;
  const double v = static_cast<double>(inv[k]) *
                   static_cast<double>(__bfloat162float(l1t[static_cast<size_t>(j) * K + k]));
  const __nv_bfloat16 hi = bf16_from_f64(v);
  l1st[static_cast<size_t>(j) * K + k] = hi;
  l1st[static_cast<size_t>(r_pad + j) * K + k] = bf16_from_f64(v - static_cast<double>(__bfloat162float(hi)));
}

// The up-projection operand of the GEMM's tail: [L2^T | L2^T] (N x 2 r_pad), so
// that one MMA over K = 2 r_pad adds (hi + lo) L2 for X_hat L1 = hi + lo.
// l2t2 = scale * [L2^T | L2^T]; scale is a power of two (the weight prescale,
// 1 without it), so the bf16 products are exact.
__global__ void dup_l2_kernel(const __nv_bfloat16* __restrict__ l2t, int N, int r_pad, float scale,
                              __nv_bfloat16* __restrict__ l2t2) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  for (int j = 0; j < r_pad; ++j) {
    const __nv_bfloat16 v =
        __float2bfloat16_rn(__fmul_rn(__bfloat162float(l2t[static_cast<size_t>(n) * r_pad + j]), scale));
    l2t2[static_cast<size_t>(n) * 2 * r_pad + j] = v;
    l2t2[static_cast<size_t>(n) * 2 * r_pad + r_pad + j] = v;
  }
}

// R[k, n] = W_hat[k, n] - sum_j L1[k, j] L2[j, n] with the bf16 factors, in fp64,
// rounded to fp32.
__global__ void residual_kernel(const double* __restrict__ What,
                                const __nv_bfloat16* __restrict__ l1t,
                                const __nv_bfloat16* __restrict__ l2t, int K, int N, int r,
                                int r_pad, float* __restrict__ R) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int k = blockIdx.y;
  if (n >= N) return;
  double acc = What[static_cast<size_t>(k) * N + n];
  for (int j = 0; j < r; ++j)
    acc -= static_cast<double>(__bfloat162float(l1t[static_cast<size_t>(j) * K + k])) *
           static_cast<double>(__bfloat162float(l2t[static_cast<size_t>(n) * r_pad + j]));
  R[static_cast<size_t>(k) * N + n] = static_cast<float>(acc);
}

// Quantize R (K x N fp32) along K for each output column n.
// NVFP4: one thread per (n, group of 16): codes N x K/2, scales in 512-byte atoms
//        (128 columns x 4 groups; byte (n % 32) * 16 + (n % 128 / 32) * 4 + g % 4).
// INT4 : one thread per (n, group of 64): int8 codes N x K, fp16 scales [K/64][N_pad].
// pre: the power-of-two weight prescale (1 without it); R * pre is exact.
__global__ void quant_weight_nvfp4_kernel(const float* __restrict__ R, int K, int N, int sf_kcols,
                                          float pre, uint8_t* __restrict__ codes,
                                          uint8_t* __restrict__ sf) {
  __shared__ float rcp_tab[128];
  fill_e4m3_rcp_table(rcp_tab, threadIdx.x, blockDim.x);
  __syncthreads();
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int g = blockIdx.y;
  if (n >= N) return;
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(R[static_cast<size_t>(16 * g + i) * N + n], pre);
  uint32_t cw[2];
  const uint32_t s8 = quant16_nvfp4(v, cw, rcp_tab);
  uint32_t* dst = reinterpret_cast<uint32_t*>(codes + static_cast<size_t>(n) * (K / 2) + 8 * g);
  dst[0] = cw[0];
  dst[1] = cw[1];
  uint8_t* atom = sf + (static_cast<size_t>(n / 128) * sf_kcols + g / 4) * 512;
  atom[(n & 31) * 16 + ((n & 127) >> 5) * 4 + (g & 3)] = static_cast<uint8_t>(s8);
}

// The weight scale atoms regrouped for the 192-column pair GEMM tiles: atom slot
// 2 nb + a (a = 0, 1) of K step kc holds the scales of weight columns
// nb * 192 + 128 a .. + 127 in the atom layout above (columns past the tile or
// past N hold 0), so that a tile's scales start at an atom boundary.  One
// thread per byte of the output, [2 * n_tiles][sf_kcols][512].
__global__ void pair192_scale_atoms_kernel(const uint8_t* __restrict__ sf, int N, int sf_kcols, int n_tiles,
                                           uint8_t* __restrict__ out) {
  const size_t total = static_cast<size_t>(2 * n_tiles) * sf_kcols * 512;
  const size_t o = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (o >= total) return;
  const int i = static_cast<int>(o % 512);
  const int kc = static_cast<int>((o / 512) % sf_kcols);
  const int ts = static_cast<int>(o / (512 * static_cast<size_t>(sf_kcols)));
  const int n = i / 16 + 32 * ((i % 16) / 4);   // column within the atom
  const int g = i % 4;
  const int nt = 128 * (ts % 2) + n;            // column within the 192-wide tile
  const int c = (ts / 2) * 192 + nt;
  uint8_t v = 0;
  if (nt < 192 && c < N)
    v = sf[(static_cast<size_t>(c / 128) * sf_kcols + kc) * 512 + (c % 32) * 16 + ((c % 128) / 32) * 4 + g];
  out[o] = v;
}

__global__ void quant_weight_int4_kernel(const float* __restrict__ R, int K, int N, int N_pad,
                                         uint8_t* __restrict__ codes, uint16_t* __restrict__ sf) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int g = blockIdx.y;
  if (n >= N) return;
  float amax = 0.f;
  for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fabsf(R[static_cast<size_t>(64 * g + i) * N + n]));
  const uint16_t sh = int4_scale_bits(amax);
  const float sd = __half2float(__ushort_as_half(sh));
  const float inv = sd == 0.f ? 0.f : __frcp_rn(sd);
  // 64 codes -> 32 bytes, element 2i in the low nibble (4-bit two's complement)
  uint32_t wd[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    uint32_t w = 0;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const float v = R[static_cast<size_t>(64 * g + 8 * e + b) * N + n];
      const uint32_t c = sd == 0.f ? 0u : static_cast<uint32_t>(int4_code(v, inv)) & 0xFu;
      w |= c << (4 * b);
    }
    wd[e] = w;
  }
  uint4* dst = reinterpret_cast<uint4*>(codes + static_cast<size_t>(n) * (K / 2) + 32 * g);
  dst[0] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
  dst[1] = make_uint4(wd[4], wd[5], wd[6], wd[7]);
  sf[static_cast<size_t>(g) * N_pad + n] = sh;
}

// The INT4 GEMM's per-column scale, derived from the fp16 weight scales:
// s_w / 16 for group g and column n (exact: an fp16 value times 2^-4).  The
// GEMM reads the partial as 16 P (its weight operand is 16 q) and scales it by
// s_x * (s_w / 16).
__global__ void int4_column_scales_kernel(const uint16_t* __restrict__ sf, size_t count, float* __restrict__ sw16) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;   // g * N_pad + n
  if (i >= count) return;
  sw16[i] = __half2float(__ushort_as_half(sf[i])) * 0.0625f;
}

// FP4 g32: one E4M3 scale per 32 values of K, stored in both 16-value slots of
// the scale atom so the NVFP4 GEMM (block16) applies it to both halves.
__global__ void quant_weight_fp4g32_kernel(const float* __restrict__ R, int K, int N, int sf_kcols,
                                           float pre, uint8_t* __restrict__ codes,
                                           uint8_t* __restrict__ sf) {
  __shared__ float rcp_tab[128];
  fill_e4m3_rcp_table(rcp_tab, threadIdx.x, blockDim.x);
  __syncthreads();
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int g = blockIdx.y;                  // group of 32
  if (n >= N) return;
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(R[static_cast<size_t>(32 * g + i) * N + n], pre);
  uint32_t cw[4];
  const uint32_t s8 = quant32_fp4(v, cw, rcp_tab);
  uint4* dst = reinterpret_cast<uint4*>(codes + static_cast<size_t>(n) * (K / 2) + 16 * g);
  *dst = make_uint4(cw[0], cw[1], cw[2], cw[3]);
  uint8_t* atom = sf + (static_cast<size_t>(n / 128) * sf_kcols + g / 2) * 512;
  uint8_t* slot = atom + (n & 31) * 16 + ((n & 127) >> 5) * 4 + 2 * (g & 1);
  slot[0] = static_cast<uint8_t>(s8);
  slot[1] = static_cast<uint8_t>(s8);
}

// ------------------------------------------------------------ refinement ---
// Iterative update of the low-rank branch (SVDQuant paper, Sec. 4.2, last
// paragraph): the part of W_hat the quantized residual misses,
// E = W_hat - deq(Q(R)), is decomposed again, and the iterate with the
// smallest ||W_hat - L1 L2 - deq(Q(R))||_F is kept.

// deq(Q(R))[k, n] from the handle's codes and scales (fmt: 0 NVFP4, 1 INT4,
// 2 FP4 g32 -- whose scale sits in both 16-value slots, so the block-of-16
// lookup serves it too).
// post: 2^-e of the weight prescale (FP4 formats; 1 without it).
__device__ __forceinline__ double deq_weight(int fmt, const uint8_t* __restrict__ codes,
                                             const uint8_t* __restrict__ sf, int K, int N_pad,
                                             int sf_kcols, double post, int k, int n) {
  if (fmt == 1) {   // packed 4-bit two's complement, fp16 scale per 64
    const uint8_t b = codes[static_cast<size_t>(n) * (K / 2) + k / 2];
    const int c = static_cast<int>((k & 1) ? (b >> 4) : (b & 15u));
    const uint16_t sh = reinterpret_cast<const uint16_t*>(sf)[static_cast<size_t>(k / 64) * N_pad + n];
    return static_cast<double>(c >= 8 ? c - 16 : c) * static_cast<double>(__half2float(__ushort_as_half(sh)));
  }
  if (fmt == 3) {   // W8A8: one fp32 scale per output channel
    const int8_t q = reinterpret_cast<const int8_t*>(codes)[static_cast<size_t>(n) * K + k];
    return static_cast<double>(__fmul_rn(static_cast<float>(q), reinterpret_cast<const float*>(sf)[n]));
  }
  const uint8_t b = codes[static_cast<size_t>(n) * (K / 2) + k / 2];
  const uint32_t c = (k & 1) ? (b >> 4) : (b & 15u);
  const int g = k / 16;
  const uint8_t s8 = sf[(static_cast<size_t>(n / 128) * sf_kcols + g / 4) * 512 + (n & 31) * 16 +
                        ((n & 127) >> 5) * 4 + (g & 3)];
  return static_cast<double>(e2m1_value(c)) * static_cast<double>(e4m3_value(s8)) * post;
}

// E = W_hat - deq(Q(R)), fp64 K x N.
__global__ void refine_target_kernel(const double* __restrict__ What, int fmt,
                                     const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf,
                                     int K, int N, int N_pad,
                                     int sf_kcols, double post, double* __restrict__ E) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int k = blockIdx.y;
  if (n >= N) return;
  const size_t i = static_cast<size_t>(k) * N + n;
  E[i] = What[i] - deq_weight(fmt, codes, sf, K, N_pad, sf_kcols, post, k, n);
}

// *sum += sum over the block's elements of (W_hat - L1 L2 - deq(Q(R)))^2, fp64.
__global__ void refine_error_kernel(const double* __restrict__ What,
                                    const __nv_bfloat16* __restrict__ l1t,
                                    const __nv_bfloat16* __restrict__ l2t, int r, int r_pad, int fmt,
                                    const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf,
                                    int K, int N, int N_pad,
                                    int sf_kcols, double post, double* __restrict__ sum) {
  __shared__ double part[8];
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int k = blockIdx.y;
  double d2 = 0.0;
  if (n < N) {
    double acc = What[static_cast<size_t>(k) * N + n];
    for (int j = 0; j < r; ++j)
      acc -= static_cast<double>(__bfloat162float(l1t[static_cast<size_t>(j) * K + k])) *
             static_cast<double>(__bfloat162float(l2t[static_cast<size_t>(n) * r_pad + j]));
    acc -= deq_weight(fmt, codes, sf, K, N_pad, sf_kcols, post, k, n);
    d2 = acc * acc;
  }
  for (int o = 16; o > 0; o >>= 1) d2 += __shfl_xor_sync(0xffffffffu, d2, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = d2;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += part[w];
    atomicAdd(sum, t);
  }
}

// W8A8 weights (SVDQuant paper, Sec. 5.1, 8-bit setting): per output channel n,
// s = max_k |R[k,n]| / 127 (IEEE fp32), codes clamp(rint_even(R * RN(1/s)), -127, 127)
// stored N x K int8; s = 0 gives zero codes.  One thread per column.
__global__ void quant_weight_w8_kernel(const float* __restrict__ R, int K, int N,
                                       int8_t* __restrict__ codes, float* __restrict__ sw) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  float amax = 0.0f;
  for (int k = 0; k < K; ++k) amax = fmaxf(amax, fabsf(R[static_cast<size_t>(k) * N + n]));
  const float s = __fdiv_rn(amax, 127.0f);
  const float inv = s == 0.0f ? 0.0f : __frcp_rn(s);
  for (int k = 0; k < K; ++k) {
    const int q = max(-127, min(127, __float2int_rn(__fmul_rn(R[static_cast<size_t>(k) * N + n], inv))));
    codes[static_cast<size_t>(n) * K + k] = static_cast<int8_t>(q);
  }
  sw[n] = s;
}

// *out = max(*out, max |R|) as the bits of a non-negative float (which order
// like the unsigned integers); *out starts at 0.  Grid-stride over n values.
__global__ void absmax_f32_kernel(const float* __restrict__ R, size_t n, unsigned int* __restrict__ out) {
  float m = 0.0f;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    m = fmaxf(m, fabsf(R[i]));
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(out, __float_as_uint(m));
}

}  // namespace svdq
