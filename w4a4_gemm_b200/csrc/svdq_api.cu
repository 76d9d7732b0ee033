// svdq_api.cu -- host side of the C ABI declared in include/svdq.h.
//
// One translation unit holds every kernel of the library (they share the
// sticky device error word), the tensor-map set-up, argument checking,
// launch configuration, weight preparation and the debug exports.
#include <cublas_v2.h>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cusolverDn.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <utility>
#include <mutex>
#include <vector>

#include "../../include/svdq.h"
#include "gemm_int4.cuh"
#include "gemm_nvfp4.cuh"
#include "gemm_nvfp4_pair.cuh"
#include "gemm_w8a8.cuh"
#include "peak.cuh"
#include "prepare.cuh"
#include "quant_act.cuh"
#include "svdq_formats.cuh"
#include "svdq_ptx.cuh"

using namespace svdq;

// E2M1 codes with E4M3 scales in the tcgen05 atom layout: NVFP4 (a scale per
// 16 values) and FP4 g32 (a scale per 32, stored twice, once per 16).
inline bool is_fp4(int fmt) { return fmt == SVDQ_NVFP4 || fmt == SVDQ_FP4G32; }

struct svdq_weights {
  int device = 0;
  int fmt = 0, K = 0, N = 0, rank = 0, r_pad = 0;
  int K_pad = 0;       // K rounded up to 256 (scale-atom columns)
  int N_pad = 0;       // N rounded up to 256
  int sf_kcols = 0;    // K_pad / 64
  float* inv_lambda = nullptr;
  float* lambda = nullptr;
  uint8_t* wcodes = nullptr;  // NVFP4, FP4 g32, INT4: N x K/2 packed (element 2i low nibble); W8A8: N x K int8
  uint8_t* wsf = nullptr;     // NVFP4: atoms [N_pad/128][sf_kcols][512]; INT4: fp16 [K/64][N_pad]
  uint8_t* wsf192 = nullptr;  // FP4: the same atoms regrouped per 192-column tile [2 n192][sf_kcols][512]
  int n192 = 0;               // FP4: 192-column tiles of N
  float* wsw16 = nullptr;     // INT4: s_w / 16 per group and column [K/64][N_pad], read by the GEMM
  __nv_bfloat16* l1t = nullptr;  // r_pad x K
  __nv_bfloat16* l1st = nullptr; // 2 r_pad x K: (diag(1/lambda) L1)^T as hi rows then lo rows, read by
                                 // the activation kernel
  __nv_bfloat16* l2t = nullptr;  // N x r_pad
  __nv_bfloat16* l2t2 = nullptr; // N x 2 r_pad: [L2^T | L2^T], the tail MMA's B operand
  __nv_bfloat16* bias = nullptr;
  CUtensorMap tm_b, tm_l1t, tm_l2t;
  CUtensorMap tm_b_half, tm_l2t_half, tm_sfb;   // FP4 CTA-pair GEMM: 128-row boxes, scale atoms
  CUtensorMap tm_b_96, tm_l2t_96, tm_sfb192;    // FP4 CTA-pair GEMM with 192-column tiles
  double refine_err0 = -1.0, refine_err = -1.0;   // weight error: SVD start, kept iterate
  unsigned flags = 0;  // SVDQ_WEIGHT_POW2_PRESCALE
  int w_exp = 0;       // the codes and scales are those of R * 2^w_exp (FP4 formats)
};

namespace {

// Process-wide state is read by the hot calls from any host thread: every
// lazily set or tunable value is atomic, and one-time set-up is published with
// a release store after it is complete.
std::atomic<long long> g_budget{-1};
std::mutex g_mutex;

long long wait_budget() {
  long long b = g_budget.load(std::memory_order_acquire);
  if (b < 0) {
    std::lock_guard<std::mutex> lk(g_mutex);
    b = g_budget.load(std::memory_order_relaxed);
    if (b < 0) {
      const char* env = std::getenv("SVDQ_WAIT_BUDGET_CYCLES");
      long long v = env ? std::atoll(env) : 0;
      b = v > 0 ? v : (1LL << 31);
      g_budget.store(b, std::memory_order_release);
    }
  }
  return b;
}

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
inline int round_up(int x, int m) { return (x + m - 1) / m * m; }

int rank_padded(int r) {
  if (r <= 0) return 0;
  if (r <= 16) return 16;
  if (r <= 32) return 32;
  return round_up(r, 64);
}

#define SVDQ_CUDA(call)                                                                \
  do {                                                                                 \
    cudaError_t e_ = (call);                                                           \
    if (e_ != cudaSuccess) {                                                           \
      std::fprintf(stderr, "svdq: %s failed: %s (%s:%d)\n", #call, cudaGetErrorString(e_), \
                   __FILE__, __LINE__);                                                \
      return SVDQ_ERR_CUDA;                                                            \
    }                                                                                  \
  } while (0)

#define SVDQ_CHECK_LAUNCH() SVDQ_CUDA(cudaGetLastError())

// Launch a hot-path kernel with programmatic stream serialization: it may be
// scheduled while the previous kernel on the stream drains, does its own setup,
// and waits for that kernel (griddep_wait) before it touches memory that other
// kernels read or write.  Every kernel launched this way calls griddep_wait.
// cluster_x > 0 also groups the CTAs into 1-D clusters of that size.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.numAttrs = 1;
  if (cluster_x > 0) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  cfg.attrs = attr;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ------------------------------------------------------------ tensor maps ---
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

CUtensorMapSwizzle swizzle_for(uint32_t row_bytes) {
  if (row_bytes >= 128) return CU_TENSOR_MAP_SWIZZLE_128B;
  if (row_bytes == 64) return CU_TENSOR_MAP_SWIZZLE_64B;
  return CU_TENSOR_MAP_SWIZZLE_32B;
}

// 2-D map over a row-major [rows][cols] array of `elem` bytes per element.
int make_map(CUtensorMap* m, CUtensorMapDataType dt, size_t elem, const void* base, uint64_t cols,
             uint64_t rows, uint32_t box_cols, uint32_t box_rows, int swizzle = -1) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return SVDQ_ERR_CUDA;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * elem};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle >= 0 ? static_cast<CUtensorMapSwizzle>(swizzle)
                               : swizzle_for(static_cast<uint32_t>(box_cols * elem)),
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::fprintf(stderr, "svdq: cuTensorMapEncodeTiled failed (%d): cols=%llu rows=%llu box=%u x %u\n",
                 static_cast<int>(r), static_cast<unsigned long long>(cols),
                 static_cast<unsigned long long>(rows), box_cols, box_rows);
    return SVDQ_ERR_CUDA;
  }
  return SVDQ_OK;
}

// Map over an array of 512-byte scale atoms as [atoms][128 x 32-bit words]; a
// box is 4 consecutive atoms (one 256-wide K step of 128 rows), no swizzle.
int make_atom_map(CUtensorMap* m, const void* base, uint64_t atoms) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return SVDQ_ERR_CUDA;
  const cuuint64_t dims[2] = {128, atoms};
  const cuuint64_t strides[1] = {512};
  const cuuint32_t box[2] = {128, 4};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::fprintf(stderr, "svdq: cuTensorMapEncodeTiled failed (%d) for %llu scale atoms\n", static_cast<int>(r),
                 static_cast<unsigned long long>(atoms));
    return SVDQ_ERR_CUDA;
  }
  return SVDQ_OK;
}

// ------------------------------------------------------------ device info ---
struct DeviceInfo {
  int sms = 0;
  int pair_clusters = 0;                    // resident clusters of the CTA-pair GEMM (256-column tiles)
  int pair192_clusters = 0;                 // the same with 192-column tiles
  int qclusters[kQuantMaxSplit + 1] = {};   // resident activation-kernel clusters of size C
  std::atomic<bool> attrs_set{false};   // set (release) once every field above is filled
};
constexpr int kMaxDevices = 64;   // device ordinals the per-device tables cover
DeviceInfo g_dev[kMaxDevices];

int device_setup(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return SVDQ_ERR_CUDA;
  DeviceInfo& d = g_dev[dev];
  if (d.attrs_set.load(std::memory_order_acquire)) return SVDQ_OK;
  std::lock_guard<std::mutex> lk(g_mutex);
  if (d.attrs_set.load(std::memory_order_relaxed)) return SVDQ_OK;
  SVDQ_CUDA(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
  uint32_t qmax = 0;
  for (int rp : {0, 16, 32, 64, 128, 192, 256})
    for (int S = 1; S <= quant_stack_max(rp); S *= 2)
      for (int f = 0; f < 2; ++f) qmax = std::max(qmax, quant_smem_layout(f, rp, S).total);
  SVDQ_CUDA(cudaFuncSetAttribute(quant_act_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, qmax));
  SVDQ_CUDA(cudaFuncSetAttribute(quant_act_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, qmax));
  SVDQ_CUDA(cudaFuncSetAttribute(quant_act_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, qmax));
  SVDQ_CUDA(cudaFuncSetAttribute(quant_act_kernel<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, qmax));
  SVDQ_CUDA(cudaFuncSetAttribute(gemm_w8a8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kW8SmemBytes));
  SVDQ_CUDA(cudaFuncSetAttribute(gemm_nvfp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kGemmSmemBytes));
  SVDQ_CUDA(cudaFuncSetAttribute(gemm_nvfp4_pair_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kPairSmemBytes));
  SVDQ_CUDA(cudaFuncSetAttribute(gemm_nvfp4_pair_kernel<192>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kPair192SmemBytes));
  SVDQ_CUDA(cudaFuncSetAttribute(gemm_int4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kI4SmemBytes));
  SVDQ_CUDA(cudaFuncSetAttribute(tensor_peak_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kPeakSmemBytes));
  SVDQ_CUDA(cudaFuncSetAttribute(tensor_peak_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kPeakSmemBytes));
  // how many clusters of each size the activation kernel can keep resident
  // (GPCs do not divide evenly into clusters of 4 or 8)
  for (int C = 1; C <= kQuantMaxSplit; C *= 2) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C * d.sms);
    cfg.blockDim = dim3(kQuantThreads);
    cfg.dynamicSmemBytes = qmax;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    SVDQ_CUDA(cudaOccupancyMaxActiveClusters(&n, quant_act_kernel<1>, &cfg));
    d.qclusters[C] = n;
  }
  for (int bn : {256, 192}) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(d.sms & ~1);
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = bn == 256 ? kPairSmemBytes : kPair192SmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (bn == 256) {
      SVDQ_CUDA(cudaOccupancyMaxActiveClusters(&n, gemm_nvfp4_pair_kernel<256>, &cfg));
      d.pair_clusters = n;
    } else {
      SVDQ_CUDA(cudaOccupancyMaxActiveClusters(&n, gemm_nvfp4_pair_kernel<192>, &cfg));
      d.pair192_clusters = n;
    }
  }
  d.attrs_set.store(true, std::memory_order_release);
  return SVDQ_OK;
}

int current_device(int* dev) {
  SVDQ_CUDA(cudaGetDevice(dev));
  return device_setup(*dev);
}

// ------------------------------------------------------------ workspace ---
// Shape of the activation kernel's launch: S stacked K sub-tiles per stage
// (BM = 128 / S rows per cluster) and C CTAs per cluster splitting K.  Cost
// model, in cycles, fitted to forced launches of every shape on B200:
//   time = waves * (fixed + [C > 1] (exchange + C * per_peer)
//                   + stages per CTA * (stage + l1 * r_pad / BM))
// fixed: setup, the first stage's round trip and the XL1 epilogue; exchange and
// per_peer: the cluster barriers and the distributed-shared-memory reads of the
// peers' partial sums; stage and l1: one 128 x 64 stage, whose L1s share
// (hi and lo: 2 r_pad / BM bytes per byte of X) travels and is read with it.  Ties go to
// the smaller C, then the smaller S.
struct QuantSplit {
  int S, C;
};
constexpr double kQuantFixedCycles = 10000.0;
constexpr double kQuantExchangeCycles = 2000.0;
constexpr double kQuantPerPeerCycles = 1000.0;
constexpr double kQuantStageCycles = 800.0;
constexpr double kQuantL1Cycles = 400.0;   // refitted with the hi + lo factor (a forced-shape sweep on B200)
std::atomic<int> g_forced_split{0};      // svdq_set_quant_split: 16 S + C; 0 = automatic
std::atomic<int> g_forced_group_m{0};    // svdq_set_gemm_raster; 0 = automatic
std::atomic<int> g_forced_gemm_kind{0};  // svdq_set_gemm_kernel; 0 = automatic, 1 = one CTA, 2 = CTA pairs,
                                         // 3 = CTA pairs on 192-column tiles, 4 = 2 with whole tiles only

QuantSplit quant_split_for(int fmt, int M, int K, int r_pad, const DeviceInfo& d) {
  const int smax = r_pad > 0 ? quant_stack_max(r_pad) : 8;
  const int fs = g_forced_split.load(std::memory_order_relaxed);
  const QuantSplit f{fs / 16, fs % 16};
  if (f.S > 0 && f.S <= smax && f.C <= kQuantTileRows / f.S &&
      f.C <= (K + f.S * kQuantBK - 1) / (f.S * kQuantBK) && d.qclusters[f.C] > 0)
    return f;
  QuantSplit best{1, 1};
  double best_t = 1e300;
  for (int C = 1; C <= kQuantMaxSplit; C *= 2) {
    const int slots = d.qclusters[C] * C;   // resident CTAs in clusters of C
    if (slots <= 0) continue;
    for (int S = 1; S <= smax; S *= 2) {
      // a stack whose stage no longer leaves room for three stage buffers
      // loses the pipeline the model assumes
      if (S > 1 && quant_smem_layout(fmt, r_pad, S).stages < 3) continue;
      const int BM = kQuantTileRows / S;
      const int stages = (K + S * kQuantBK - 1) / (S * kQuantBK);
      if (C > BM || C > stages) continue;
      const long long ctas = static_cast<long long>((M + BM - 1) / BM) * C;
      const long long waves = (ctas + slots - 1) / slots;
      const int per = (stages + C - 1) / C;
      const double t = static_cast<double>(waves) *
                       (kQuantFixedCycles + (C > 1 ? kQuantExchangeCycles + C * kQuantPerPeerCycles : 0.0) +
                        per * (kQuantStageCycles + kQuantL1Cycles * 2 * r_pad / BM));
      if (t < best_t * 0.98) {
        best_t = t;
        best = {S, C};
      }
    }
  }
  return best;
}

struct ActLayout {
  int M, M_pad;
  size_t codes_off, codes_bytes, sf_off, sf_bytes, xl1_off, xl1_bytes, total;
};

ActLayout act_layout(const svdq_weights* w, int M) {
  ActLayout L;
  L.M = M;
  L.M_pad = round_up(std::max(M, 1), 128);
  L.codes_bytes = is_fp4(w->fmt) ? static_cast<size_t>(M) * w->K / 2
                                       : static_cast<size_t>(M) * w->K;
  L.sf_bytes = is_fp4(w->fmt)            ? static_cast<size_t>(L.M_pad / 128) * w->sf_kcols * 512
               : w->fmt == SVDQ_W8A8 ? static_cast<size_t>(L.M_pad) * 4          // fp32 per token
                                     : static_cast<size_t>(w->K / 64) * L.M_pad * 2;
  L.xl1_bytes = static_cast<size_t>(M) * 2 * w->r_pad * 2;   // bf16 hi | lo
  L.codes_off = 0;
  L.sf_off = align256(L.codes_bytes);
  L.xl1_off = L.sf_off + align256(L.sf_bytes);
  L.total = L.xl1_off + align256(L.xl1_bytes);
  return L;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int encode_weight_maps(svdq_weights* w) {
  int rc;
  if (is_fp4(w->fmt)) {
    rc = make_map(&w->tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->wcodes, w->K / 2, w->N, 128, kGemmBN);
    if (!rc) rc = make_map(&w->tm_b_half, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->wcodes, w->K / 2, w->N, 128, 128);
    if (!rc) rc = make_atom_map(&w->tm_sfb, w->wsf, static_cast<uint64_t>(w->N_pad / 128) * w->sf_kcols);
    if (!rc) rc = make_map(&w->tm_b_96, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->wcodes, w->K / 2, w->N, 128, 96);
    if (!rc) rc = make_atom_map(&w->tm_sfb192, w->wsf192, static_cast<uint64_t>(2 * w->n192) * w->sf_kcols);
  } else if (w->fmt == SVDQ_W8A8)
    rc = make_map(&w->tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->wcodes, w->K, w->N, kW8BKB, kW8BN);
  else   // INT4: the packed codes, 32 bytes (64 codes) x 128 columns per box, read by the drain warps
    rc = make_map(&w->tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w->wcodes, w->K / 2, w->N, 32, kI4BN,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc) return rc;
  if (w->r_pad > 0) {
    rc = make_map(&w->tm_l1t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w->l1st, w->K, 2 * w->r_pad, 64, w->r_pad);
    if (rc) return rc;
    const int lc = w->fmt != SVDQ_INT4 ? lr_chunk_cols(2 * w->r_pad) : i4_lr_chunk_cols(2 * w->r_pad);
    rc = make_map(&w->tm_l2t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w->l2t2, 2 * w->r_pad, w->N, lc,
                  w->fmt != SVDQ_INT4 ? kGemmBN : kI4BN);
    if (rc) return rc;
    if (is_fp4(w->fmt) &&
        (rc = make_map(&w->tm_l2t_half, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w->l2t2, 2 * w->r_pad, w->N, lc, 128)))
      return rc;
    if (is_fp4(w->fmt) &&
        (rc = make_map(&w->tm_l2t_96, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w->l2t2, 2 * w->r_pad, w->N, lc, 96)))
      return rc;
  } else {
    w->tm_l1t = w->tm_b;
    w->tm_l2t = w->tm_b;
    w->tm_l2t_half = w->tm_b;
    w->tm_l2t_96 = w->tm_b;
  }
  return SVDQ_OK;
}

void free_weights(svdq_weights* w) {
  if (!w) return;
  cudaFree(w->inv_lambda);
  cudaFree(w->lambda);
  cudaFree(w->wcodes);
  cudaFree(w->wsf);
  cudaFree(w->wsf192);
  cudaFree(w->wsw16);
  cudaFree(w->l1t);
  cudaFree(w->l1st);
  cudaFree(w->l2t);
  cudaFree(w->l2t2);
  cudaFree(w->bias);
  delete w;
}

int check_shape(int fmt, int K, int N, int rank) {
  if (fmt != SVDQ_NVFP4 && fmt != SVDQ_INT4 && fmt != SVDQ_FP4G32 && fmt != SVDQ_W8A8)
    return SVDQ_ERR_INVALID_ARG;
  if (K <= 0 || N <= 0 || K % 64 != 0 || N % 16 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (rank < 0 || rank > 256 || rank > std::min(K, N)) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  return SVDQ_OK;
}

// Allocate the quantized-weight buffers and the (zeroed) factor layouts.
int alloc_weights(svdq_weights* w, cudaStream_t st) {
  w->K_pad = round_up(w->K, 256);
  w->N_pad = round_up(w->N, 256);
  w->sf_kcols = w->K_pad / 64;
  w->r_pad = rank_padded(w->rank);
  const size_t codes = w->fmt != SVDQ_W8A8 ? static_cast<size_t>(w->N) * w->K / 2
                                            : static_cast<size_t>(w->N) * w->K;
  const size_t sfb = is_fp4(w->fmt)            ? static_cast<size_t>(w->N_pad / 128) * w->sf_kcols * 512
                     : w->fmt == SVDQ_W8A8 ? static_cast<size_t>(w->N_pad) * 4   // fp32 per channel
                                           : static_cast<size_t>(w->K / 64) * w->N_pad * 2;
  // 1/lambda is read in 512-value blocks by the activation kernel: zero-pad it
  const size_t il_bytes = static_cast<size_t>(round_up(w->K, 512)) * sizeof(float);
  if (cudaMalloc(&w->inv_lambda, il_bytes) != cudaSuccess ||
      cudaMalloc(&w->lambda, w->K * sizeof(float)) != cudaSuccess ||
      cudaMalloc(&w->wcodes, codes) != cudaSuccess || cudaMalloc(&w->wsf, sfb) != cudaSuccess)
    return SVDQ_ERR_ALLOC;
  SVDQ_CUDA(cudaMemsetAsync(w->inv_lambda, 0, il_bytes, st));
  SVDQ_CUDA(cudaMemsetAsync(w->wsf, 0, sfb, st));
  if (is_fp4(w->fmt)) {
    w->n192 = (w->N + 191) / 192;
    const size_t sf192 = static_cast<size_t>(2 * w->n192) * w->sf_kcols * 512;
    if (cudaMalloc(&w->wsf192, sf192) != cudaSuccess) return SVDQ_ERR_ALLOC;
    SVDQ_CUDA(cudaMemsetAsync(w->wsf192, 0, sf192, st));
  }
  if (w->fmt == SVDQ_INT4) {
    const size_t sw16 = static_cast<size_t>(w->K / 64) * w->N_pad * sizeof(float);
    if (cudaMalloc(&w->wsw16, sw16) != cudaSuccess) return SVDQ_ERR_ALLOC;
    SVDQ_CUDA(cudaMemsetAsync(w->wsw16, 0, sw16, st));
  }
  if (w->r_pad > 0) {
    if (cudaMalloc(&w->l1t, static_cast<size_t>(w->r_pad) * w->K * 2) != cudaSuccess ||
        cudaMalloc(&w->l1st, static_cast<size_t>(2 * w->r_pad) * w->K * 2) != cudaSuccess ||
        cudaMalloc(&w->l2t, static_cast<size_t>(w->N) * w->r_pad * 2) != cudaSuccess)
      return SVDQ_ERR_ALLOC;
    SVDQ_CUDA(cudaMemsetAsync(w->l1t, 0, static_cast<size_t>(w->r_pad) * w->K * 2, st));
    SVDQ_CUDA(cudaMemsetAsync(w->l1st, 0, static_cast<size_t>(2 * w->r_pad) * w->K * 2, st));
    SVDQ_CUDA(cudaMemsetAsync(w->l2t, 0, static_cast<size_t>(w->N) * w->r_pad * 2, st));
  }
  return SVDQ_OK;
}

struct DeviceBuf {
  void* p = nullptr;
  ~DeviceBuf() { if (p) cudaFree(p); }
  bool alloc(size_t n) { return cudaMalloc(&p, n) == cudaSuccess; }
  template <class T> T* as() const { return static_cast<T*>(p); }
};

// The optional power-of-two prescale of the weight residual: the largest e
// with 2^e * s_max <= 448 (the top of the E4M3 range), s_max = fp32(max|R| / 6)
// the largest group scale before rounding; 0 for a zero residual.  Computed
// from the bits: s_max = f 2^q with 0.5 <= f < 1 and 448 = 0.875 * 2^9.
int prescale_exponent(float amax) {
  const float s_max = amax / 6.0f;
  if (!(s_max > 0.0f)) return 0;
  int q = 0;
  const float f = std::frexp(s_max, &q);
  const int e = f <= 0.875f ? 9 - q : 8 - q;
  return std::max(-64, std::min(64, e));
}

// Derived operand of the tail MMA: l2t2 = 2^w_exp [L2^T | L2^T].
int build_l2t2(svdq_weights* w, cudaStream_t st) {
  if (w->rank == 0 || w->l2t2 == nullptr) return SVDQ_OK;
  dup_l2_kernel<<<(w->N + 255) / 256, 256, 0, st>>>(w->l2t, w->N, w->r_pad, std::ldexp(1.0f, w->w_exp),
                                                    w->l2t2);
  SVDQ_CHECK_LAUNCH();
  return SVDQ_OK;
}

// Scale layouts derived from the weight scales in w->wsf, redone whenever
// those change (quantization, or a refinement restoring an earlier iterate):
// FP4 formats: the atoms regrouped per 192-column tile of the pair GEMM;
// INT4: the GEMM's s_w / 16 per group and column.
int derive_scale_layouts(svdq_weights* w, cudaStream_t st) {
  if (w->fmt == SVDQ_INT4) {
    const size_t n = static_cast<size_t>(w->K / 64) * w->N_pad;
    int4_column_scales_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(
        reinterpret_cast<const uint16_t*>(w->wsf), n, w->wsw16);
    SVDQ_CHECK_LAUNCH();
  }
  if (is_fp4(w->fmt)) {
    const size_t sf192 = static_cast<size_t>(2 * w->n192) * w->sf_kcols * 512;
    pair192_scale_atoms_kernel<<<static_cast<unsigned>((sf192 + 255) / 256), 256, 0, st>>>(
        w->wsf, w->N, w->sf_kcols, w->n192, w->wsf192);
    SVDQ_CHECK_LAUNCH();
  }
  return SVDQ_OK;
}

int quantize_residual(svdq_weights* w, const float* R, cudaStream_t st) {
  const dim3 blk(128);
  const int e_old = w->w_exp;
  w->w_exp = 0;
  if ((w->flags & SVDQ_WEIGHT_POW2_PRESCALE) && is_fp4(w->fmt)) {
    DeviceBuf amax;
    if (!amax.alloc(sizeof(unsigned))) return SVDQ_ERR_ALLOC;
    SVDQ_CUDA(cudaMemsetAsync(amax.p, 0, sizeof(unsigned), st));
    absmax_f32_kernel<<<4 * 148, 256, 0, st>>>(R, static_cast<size_t>(w->K) * w->N, amax.as<unsigned>());
    SVDQ_CHECK_LAUNCH();
    unsigned bits = 0;
    SVDQ_CUDA(cudaMemcpyAsync(&bits, amax.p, sizeof bits, cudaMemcpyDeviceToHost, st));
    SVDQ_CUDA(cudaStreamSynchronize(st));
    float a;
    std::memcpy(&a, &bits, sizeof a);
    w->w_exp = prescale_exponent(a);
  }
  const float pre = std::ldexp(1.0f, w->w_exp);
  if (w->fmt == SVDQ_NVFP4) {
    const dim3 grid((w->N + 127) / 128, w->K / 16);
    quant_weight_nvfp4_kernel<<<grid, blk, 0, st>>>(R, w->K, w->N, w->sf_kcols, pre, w->wcodes, w->wsf);
  } else if (w->fmt == SVDQ_FP4G32) {
    const dim3 grid((w->N + 127) / 128, w->K / 32);
    quant_weight_fp4g32_kernel<<<grid, blk, 0, st>>>(R, w->K, w->N, w->sf_kcols, pre, w->wcodes, w->wsf);
  } else if (w->fmt == SVDQ_W8A8) {
    quant_weight_w8_kernel<<<(w->N + 127) / 128, blk, 0, st>>>(R, w->K, w->N,
                                                                reinterpret_cast<int8_t*>(w->wcodes),
                                                                reinterpret_cast<float*>(w->wsf));
  } else {
    const dim3 grid((w->N + 127) / 128, w->K / 64);
    quant_weight_int4_kernel<<<grid, blk, 0, st>>>(R, w->K, w->N, w->N_pad, w->wcodes,
                                                   reinterpret_cast<uint16_t*>(w->wsf));
  }
  SVDQ_CHECK_LAUNCH();
  if (int rc = derive_scale_layouts(w, st)) return rc;
  if (w->w_exp != e_old) return build_l2t2(w, st);   // the tail carries the same 2^e
  return SVDQ_OK;
}

// The derived operands the kernels read: l1st = (diag(1/lambda) L1)^T as a bf16
// pair hi | lo and l2t2 = [L2^T | L2^T], from the current l1t, l2t and inv_lambda.
int refold_l1(svdq_weights* w, cudaStream_t st) {
  if (w->rank == 0) return SVDQ_OK;
  cudaFree(w->l2t2);
  w->l2t2 = nullptr;
  if (cudaMalloc(&w->l2t2, static_cast<size_t>(w->N) * 2 * w->r_pad * 2) != cudaSuccess)
    return SVDQ_ERR_ALLOC;
  if (int rc = build_l2t2(w, st)) return rc;
  fold_l1_kernel<<<dim3((w->K + 255) / 256, w->rank), 256, 0, st>>>(w->l1t, w->inv_lambda, w->K,
                                                                     w->rank, w->r_pad, w->l1st);
  SVDQ_CHECK_LAUNCH();
  return SVDQ_OK;
}

int copy_bias(svdq_weights* w, const void* bias, cudaStream_t st) {
  if (bias == nullptr) return SVDQ_OK;
  if (cudaMalloc(&w->bias, static_cast<size_t>(w->N) * 2) != cudaSuccess) return SVDQ_ERR_ALLOC;
  SVDQ_CUDA(cudaMemcpyAsync(w->bias, bias, static_cast<size_t>(w->N) * 2, cudaMemcpyDeviceToDevice, st));
  return SVDQ_OK;
}

int do_append_lora(svdq_weights* w, const void* A, const void* B, int rl, cudaStream_t st) {
  if (rl <= 0) return SVDQ_OK;
  const int r_old = w->rank, rp_old = w->r_pad;
  const int r_new = r_old + rl;
  if (r_new > 256 || r_new > std::min(w->K, w->N)) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  const int rp_new = rank_padded(r_new);
  __nv_bfloat16 *l1t = nullptr, *l1st = nullptr, *l2t = nullptr;
  if (cudaMalloc(&l1t, static_cast<size_t>(rp_new) * w->K * 2) != cudaSuccess) return SVDQ_ERR_ALLOC;
  if (cudaMalloc(&l1st, static_cast<size_t>(2 * rp_new) * w->K * 2) != cudaSuccess) {
    cudaFree(l1t);
    return SVDQ_ERR_ALLOC;
  }
  if (cudaMalloc(&l2t, static_cast<size_t>(w->N) * rp_new * 2) != cudaSuccess) {
    cudaFree(l1t);
    cudaFree(l1st);
    return SVDQ_ERR_ALLOC;
  }
  cudaMemsetAsync(l1t, 0, static_cast<size_t>(rp_new) * w->K * 2, st);
  cudaMemsetAsync(l1st, 0, static_cast<size_t>(2 * rp_new) * w->K * 2, st);
  cudaMemsetAsync(l2t, 0, static_cast<size_t>(w->N) * rp_new * 2, st);
  if (r_old > 0) {
    const size_t n1 = static_cast<size_t>(r_old) * w->K;
    widen_l1_kernel<<<static_cast<unsigned>((n1 + 255) / 256), 256, 0, st>>>(w->l1t, w->K, r_old, l1t);
    widen_l2_kernel<<<(w->N + 255) / 256, 256, 0, st>>>(w->l2t, w->N, r_old, rp_old, rp_new, l2t);
  }
  lora_l1_kernel<<<dim3((w->K + 255) / 256, rl), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(A), w->lambda, w->K, rl, r_old, l1t);
  layout_l2_kernel<<<dim3((w->N + 255) / 256, rl), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(B), w->N, rl, r_old, rp_new, l2t);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) {
    cudaFree(l1t);
    cudaFree(l1st);
    cudaFree(l2t);
    std::fprintf(stderr, "svdq: LoRA fold failed: %s\n", cudaGetErrorString(e));
    return SVDQ_ERR_CUDA;
  }
  cudaFree(w->l1t);
  cudaFree(w->l1st);
  cudaFree(w->l2t);
  w->l1t = l1t;
  w->l1st = l1st;
  w->l2t = l2t;
  w->rank = r_new;
  w->r_pad = rp_new;
  int rc = refold_l1(w, st);
  if (rc == SVDQ_OK && cudaStreamSynchronize(st) != cudaSuccess) rc = SVDQ_ERR_CUDA;
  if (rc) return rc;
  return encode_weight_maps(w);
}

// Optimal rank-r factors of W_hat (fp64, K x N row-major) into w->l1t / w->l2t:
// eigen-decomposition of the smaller Gram matrix (cuBLAS DSYRK + cuSOLVER DSYEVD).
int lowrank_factors(svdq_weights* w, const double* What, cudaStream_t st) {
  const int K = w->K, N = w->N, r = w->rank;
  const bool left = K <= N;                 // G = W_hat W_hat^T (K x K), else W_hat^T W_hat
  const int d = left ? K : N;
  DeviceBuf G, ev, info, work;
  if (!G.alloc(static_cast<size_t>(d) * d * 8) || !ev.alloc(static_cast<size_t>(d) * 8) ||
      !info.alloc(sizeof(int)))
    return SVDQ_ERR_ALLOC;
  cublasHandle_t cb = nullptr;
  cusolverDnHandle_t cs = nullptr;
  int rc = SVDQ_OK;
  if (cublasCreate(&cb) != CUBLAS_STATUS_SUCCESS) return SVDQ_ERR_LIBRARY;
  if (cusolverDnCreate(&cs) != CUSOLVER_STATUS_SUCCESS) {
    cublasDestroy(cb);
    return SVDQ_ERR_LIBRARY;
  }
  cublasSetStream(cb, st);
  cusolverDnSetStream(cs, st);
  const double one = 1.0, zero = 0.0;
  // W_hat (row-major K x N) is the column-major N x K matrix A = W_hat^T.
  cublasStatus_t bs = left
      ? cublasDsyrk(cb, CUBLAS_FILL_MODE_LOWER, CUBLAS_OP_T, K, N, &one, What, N, &zero, G.as<double>(), K)
      : cublasDsyrk(cb, CUBLAS_FILL_MODE_LOWER, CUBLAS_OP_N, N, K, &one, What, N, &zero, G.as<double>(), N);
  if (bs != CUBLAS_STATUS_SUCCESS) rc = SVDQ_ERR_LIBRARY;
  int lwork = 0;
  if (!rc && cusolverDnDsyevd_bufferSize(cs, CUSOLVER_EIG_MODE_VECTOR, CUBLAS_FILL_MODE_LOWER, d,
                                         G.as<double>(), d, ev.as<double>(), &lwork) !=
                 CUSOLVER_STATUS_SUCCESS)
    rc = SVDQ_ERR_LIBRARY;
  if (!rc && !work.alloc(static_cast<size_t>(std::max(lwork, 1)) * 8)) rc = SVDQ_ERR_ALLOC;
  if (!rc && cusolverDnDsyevd(cs, CUSOLVER_EIG_MODE_VECTOR, CUBLAS_FILL_MODE_LOWER, d, G.as<double>(),
                              d, ev.as<double>(), work.as<double>(), lwork, info.as<int>()) !=
                 CUSOLVER_STATUS_SUCCESS)
    rc = SVDQ_ERR_LIBRARY;
  if (!rc) {
    int h_info = 0;
    if (cudaMemcpyAsync(&h_info, info.p, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      rc = SVDQ_ERR_CUDA;
    else if (h_info != 0)
      rc = SVDQ_ERR_LIBRARY;
  }
  if (!rc) {
    lowrank_l1_kernel<<<dim3((K + 127) / 128, w->r_pad), 128, 0, st>>>(
        G.as<double>(), ev.as<double>(), What, K, N, r, w->r_pad, left ? 1 : 0, w->l1t, nullptr);
    lowrank_l2_kernel<<<dim3((N + 127) / 128, w->r_pad), 128, 0, st>>>(
        G.as<double>(), ev.as<double>(), What, K, N, r, w->r_pad, left ? 1 : 0, w->l2t);
    if (cudaGetLastError() != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess)
      rc = SVDQ_ERR_CUDA;
  }
  cusolverDnDestroy(cs);
  cublasDestroy(cb);
  return rc;
}

// ||W_hat - L1 L2 - deq(Q(R))||_F of the handle's current branch and codes.
int weight_error(svdq_weights* w, const double* What, double* err_dev, double* out, cudaStream_t st) {
  SVDQ_CUDA(cudaMemsetAsync(err_dev, 0, sizeof(double), st));
  refine_error_kernel<<<dim3((w->N + 255) / 256, w->K), 256, 0, st>>>(
      What, w->l1t, w->l2t, w->rank, w->r_pad, w->fmt, w->wcodes, w->wsf, w->K, w->N,
      w->N_pad, w->sf_kcols, std::ldexp(1.0, -w->w_exp), err_dev);
  SVDQ_CHECK_LAUNCH();
  double h = 0.0;
  SVDQ_CUDA(cudaMemcpyAsync(&h, err_dev, sizeof(double), cudaMemcpyDeviceToHost, st));
  SVDQ_CUDA(cudaStreamSynchronize(st));
  *out = std::sqrt(h);
  return SVDQ_OK;
}

// Iterative update of the low-rank branch (SVDQuant paper, Sec. 4.2, last
// paragraph): iters times, factor E = W_hat - deq(Q(R)), R = W_hat - L1 L2,
// requantize; keep the iterate with the smallest weight error.  R is scratch.
int refine_branch(svdq_weights* w, const double* What, float* R, int iters, cudaStream_t st) {
  const size_t KN = static_cast<size_t>(w->K) * w->N;
  const size_t l1b = static_cast<size_t>(w->r_pad) * w->K * 2, l2b = static_cast<size_t>(w->N) * w->r_pad * 2;
  const size_t cb = w->fmt != SVDQ_W8A8 ? KN / 2 : KN;
  const size_t sfb = is_fp4(w->fmt)            ? static_cast<size_t>(w->N_pad / 128) * w->sf_kcols * 512
                     : w->fmt == SVDQ_W8A8 ? static_cast<size_t>(w->N_pad) * 4
                                           : static_cast<size_t>(w->K / 64) * w->N_pad * 2;
  DeviceBuf E, err, b_l1, b_l2, b_codes, b_sf;
  if (!E.alloc(KN * 8) || !err.alloc(sizeof(double)) || !b_l1.alloc(l1b) || !b_l2.alloc(l2b) ||
      !b_codes.alloc(cb) || !b_sf.alloc(sfb))
    return SVDQ_ERR_ALLOC;
  auto save = [&](bool to_best) -> int {
    auto cp = [&](void* best, void* cur, size_t n) {
      return to_best ? cudaMemcpyAsync(best, cur, n, cudaMemcpyDeviceToDevice, st)
                     : cudaMemcpyAsync(cur, best, n, cudaMemcpyDeviceToDevice, st);
    };
    if (cp(b_l1.p, w->l1t, l1b) != cudaSuccess || cp(b_l2.p, w->l2t, l2b) != cudaSuccess ||
        cp(b_codes.p, w->wcodes, cb) != cudaSuccess || cp(b_sf.p, w->wsf, sfb) != cudaSuccess)
      return SVDQ_ERR_CUDA;
    return SVDQ_OK;
  };
  int rc;
  double best = 0.0, e = 0.0;
  if ((rc = weight_error(w, What, err.as<double>(), &best, st))) return rc;
  w->refine_err0 = best;
  if ((rc = save(true))) return rc;
  int best_exp = w->w_exp;   // the prescale exponent the kept codes and scales were made with
  for (int t = 0; t < iters; ++t) {
    refine_target_kernel<<<dim3((w->N + 255) / 256, w->K), 256, 0, st>>>(
        What, w->fmt, w->wcodes, w->wsf, w->K, w->N, w->N_pad, w->sf_kcols,
        std::ldexp(1.0, -w->w_exp), E.as<double>());
    SVDQ_CHECK_LAUNCH();
    if ((rc = lowrank_factors(w, E.as<double>(), st))) return rc;
    residual_kernel<<<dim3((w->N + 255) / 256, w->K), 256, 0, st>>>(What, w->l1t, w->l2t, w->K, w->N,
                                                                       w->rank, w->r_pad, R);
    SVDQ_CHECK_LAUNCH();
    if ((rc = quantize_residual(w, R, st))) return rc;
    if ((rc = weight_error(w, What, err.as<double>(), &e, st))) return rc;
    if (e < best) {
      best = e;
      best_exp = w->w_exp;
      if ((rc = save(true))) return rc;
    }
  }
  if ((rc = save(false))) return rc;
  w->w_exp = best_exp;   // the caller rebuilds [L2^T | L2^T] (refold_l1) with it
  if ((rc = derive_scale_layouts(w, st))) return rc;
  w->refine_err = best;
  SVDQ_CUDA(cudaStreamSynchronize(st));
  return SVDQ_OK;
}

}  // namespace

// =========================================================================
extern "C" {

SVDQ_API const char* svdq_status_string(int s) {
  switch (s) {
    case SVDQ_OK: return "ok";
    case SVDQ_ERR_INVALID_ARG: return "invalid argument";
    case SVDQ_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case SVDQ_ERR_ALLOC: return "device allocation failed";
    case SVDQ_ERR_CUDA: return "CUDA error";
    case SVDQ_ERR_TIMEOUT: return "device wait timed out";
    case SVDQ_ERR_LIBRARY: return "cuSOLVER/cuBLAS error";
    default: return "unknown status";
  }
}

SVDQ_API int svdq_tensor_peak(int fmt, long long steps, void* stream) {
  if ((fmt != SVDQ_NVFP4 && fmt != SVDQ_INT4 && fmt != SVDQ_FP4G32 && fmt != SVDQ_W8A8) || steps < 1)
    return SVDQ_ERR_INVALID_ARG;
  int dev;
  int rc = current_device(&dev);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (is_fp4(fmt))
    tensor_peak_kernel<0><<<g_dev[dev].sms, kPeakThreads, kPeakSmemBytes, st>>>(steps, wait_budget());
  else
    tensor_peak_kernel<1><<<g_dev[dev].sms, kPeakThreads, kPeakSmemBytes, st>>>(steps, wait_budget());
  SVDQ_CHECK_LAUNCH();
  return SVDQ_OK;
}

SVDQ_API int svdq_set_gemm_kernel(int kind) {
  if (kind < 0 || kind > 4) return SVDQ_ERR_INVALID_ARG;
  g_forced_gemm_kind.store(kind, std::memory_order_relaxed);
  return SVDQ_OK;
}

SVDQ_API int svdq_set_gemm_raster(int group_m) {
  if (group_m < 0) return SVDQ_ERR_INVALID_ARG;
  g_forced_group_m.store(group_m, std::memory_order_relaxed);
  return SVDQ_OK;
}

SVDQ_API int svdq_set_quant_split(int S, int C) {
  auto pow2_le8 = [](int v) { return v == 1 || v == 2 || v == 4 || v == 8; };
  if (S == 0 && C == 0) {
    g_forced_split.store(0, std::memory_order_relaxed);
    return SVDQ_OK;
  }
  if (!pow2_le8(S) || !pow2_le8(C)) return SVDQ_ERR_INVALID_ARG;
  g_forced_split.store(16 * S + C, std::memory_order_relaxed);
  return SVDQ_OK;
}

SVDQ_API int svdq_set_wait_budget(long long cycles) {
  if (cycles <= 0) return SVDQ_ERR_INVALID_ARG;
  g_budget.store(cycles, std::memory_order_release);
  return SVDQ_OK;
}

SVDQ_API int svdq_get_error(void) {
  unsigned v = 0, z = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return -SVDQ_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&v, g_error_word, sizeof v) != cudaSuccess) return -SVDQ_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_error_word, &z, sizeof z) != cudaSuccess) return -SVDQ_ERR_CUDA;
  return static_cast<int>(v);
}

SVDQ_API int svdq_calib_absmax(const void* X, int M, int K, float* absmax, int accumulate,
                               void* stream) {
  if (X == nullptr || absmax == nullptr || M < 0 || K <= 0 || (K & 1)) return SVDQ_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!accumulate) SVDQ_CUDA(cudaMemsetAsync(absmax, 0, static_cast<size_t>(K) * 4, st));
  if (M == 0) return SVDQ_OK;
  const int pairs = K / 2;
  const int splits = std::min(64, std::max(1, M / 64));
  calib_absmax_kernel<<<dim3((pairs + 255) / 256, splits), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(X), M, K, absmax);
  SVDQ_CHECK_LAUNCH();
  return SVDQ_OK;
}

SVDQ_API int svdq_prepare_weights(const svdq_prepare_desc* d, void* stream, svdq_weights** out) {
  if (d == nullptr || out == nullptr || d->W == nullptr) return SVDQ_ERR_INVALID_ARG;
  *out = nullptr;
  int rc = check_shape(d->fmt, d->K, d->N, d->rank);
  if (rc) return rc;
  if (d->lora_rank < 0 || (d->lora_rank > 0 && (d->lora_A == nullptr || d->lora_B == nullptr)))
    return SVDQ_ERR_INVALID_ARG;
  if (d->rank + d->lora_rank > 256 || d->rank + d->lora_rank > std::min(d->K, d->N))
    return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (d->refine_iters < 0 || d->refine_iters > 64) return SVDQ_ERR_INVALID_ARG;
  if (d->flags & ~SVDQ_WEIGHT_POW2_PRESCALE) return SVDQ_ERR_INVALID_ARG;
  int dev;
  if ((rc = current_device(&dev))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  svdq_weights* w = new svdq_weights();
  w->device = dev;
  w->fmt = d->fmt;
  w->K = d->K;
  w->N = d->N;
  w->rank = d->rank;
  w->flags = d->flags;
  const int K = d->K, N = d->N;
  do {
    if ((rc = alloc_weights(w, st))) break;
    DeviceBuf wmax, What, R;
    if (!wmax.alloc(static_cast<size_t>(K) * 4) || !What.alloc(static_cast<size_t>(K) * N * 8) ||
        !R.alloc(static_cast<size_t>(K) * N * 4)) {
      rc = SVDQ_ERR_ALLOC;
      break;
    }
    const __nv_bfloat16* W = static_cast<const __nv_bfloat16*>(d->W);
    row_absmax_kernel<<<K, 256, 0, st>>>(W, K, N, wmax.as<float>());
    smoothing_kernel<<<(K + 255) / 256, 256, 0, st>>>(d->x_absmax, wmax.as<float>(), K, w->lambda,
                                                      w->inv_lambda);
    const size_t KN = static_cast<size_t>(K) * N;
    smooth_weight_kernel<<<static_cast<unsigned>((KN + 255) / 256), 256, 0, st>>>(
        W, w->lambda, K, N, What.as<double>());
    if (cudaGetLastError() != cudaSuccess) {
      rc = SVDQ_ERR_CUDA;
      break;
    }
    if (w->rank > 0 && (rc = lowrank_factors(w, What.as<double>(), st))) break;
    if ((rc = refold_l1(w, st))) break;
    residual_kernel<<<dim3((N + 255) / 256, K), 256, 0, st>>>(
        What.as<double>(), w->l1t, w->l2t, K, N, w->rank, w->r_pad, R.as<float>());
    if (cudaGetLastError() != cudaSuccess) {
      rc = SVDQ_ERR_CUDA;
      break;
    }
    if ((rc = quantize_residual(w, R.as<float>(), st))) break;
    if (d->refine_iters > 0 && w->rank > 0) {
      if ((rc = refine_branch(w, What.as<double>(), R.as<float>(), d->refine_iters, st))) break;
      if ((rc = refold_l1(w, st))) break;   // the folded factors of the kept iterate
    }
    if ((rc = copy_bias(w, d->bias, st))) break;
    if (cudaStreamSynchronize(st) != cudaSuccess) {
      rc = SVDQ_ERR_CUDA;
      break;
    }
    if ((rc = encode_weight_maps(w))) break;
    if (d->lora_rank > 0 && (rc = do_append_lora(w, d->lora_A, d->lora_B, d->lora_rank, st))) break;
  } while (false);
  if (rc) {
    free_weights(w);
    return rc;
  }
  *out = w;
  return SVDQ_OK;
}

SVDQ_API int svdq_load_weights(const svdq_parts_desc* d, void* stream, svdq_weights** out) {
  if (d == nullptr || out == nullptr || d->R == nullptr) return SVDQ_ERR_INVALID_ARG;
  *out = nullptr;
  int rc = check_shape(d->fmt, d->K, d->N, d->rank);
  if (rc) return rc;
  if (d->rank > 0 && (d->L1 == nullptr || d->L2 == nullptr)) return SVDQ_ERR_INVALID_ARG;
  if (d->flags & ~SVDQ_WEIGHT_POW2_PRESCALE) return SVDQ_ERR_INVALID_ARG;
  int dev;
  if ((rc = current_device(&dev))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  svdq_weights* w = new svdq_weights();
  w->device = dev;
  w->fmt = d->fmt;
  w->K = d->K;
  w->N = d->N;
  w->rank = d->rank;
  w->flags = d->flags;
  const int K = d->K, N = d->N;
  do {
    if ((rc = alloc_weights(w, st))) break;
    std::vector<float> ones;
    if (d->inv_lambda) {
      if (cudaMemcpyAsync(w->inv_lambda, d->inv_lambda, K * 4, cudaMemcpyDeviceToDevice, st)) {
        rc = SVDQ_ERR_CUDA;
        break;
      }
    }
    if (d->lambda) {
      if (cudaMemcpyAsync(w->lambda, d->lambda, K * 4, cudaMemcpyDeviceToDevice, st)) {
        rc = SVDQ_ERR_CUDA;
        break;
      }
    }
    if (!d->inv_lambda || !d->lambda) {
      // host-side fill: lambda = 1 / inv_lambda (or both 1)
      std::vector<float> inv(K, 1.0f), lam(K, 1.0f);
      if (d->inv_lambda &&
          cudaMemcpy(inv.data(), d->inv_lambda, K * 4, cudaMemcpyDeviceToHost) != cudaSuccess) {
        rc = SVDQ_ERR_CUDA;
        break;
      }
      for (int k = 0; k < K; ++k) lam[k] = 1.0f / inv[k];
      if (!d->inv_lambda && cudaMemcpy(w->inv_lambda, inv.data(), K * 4, cudaMemcpyHostToDevice)) {
        rc = SVDQ_ERR_CUDA;
        break;
      }
      if (!d->lambda && cudaMemcpy(w->lambda, lam.data(), K * 4, cudaMemcpyHostToDevice)) {
        rc = SVDQ_ERR_CUDA;
        break;
      }
    }
    if (w->rank > 0) {
      layout_l1_kernel<<<dim3((K + 255) / 256, w->rank), 256, 0, st>>>(
          static_cast<const __nv_bfloat16*>(d->L1), K, w->rank, 0, w->l1t);
      layout_l2_kernel<<<dim3((N + 255) / 256, w->rank), 256, 0, st>>>(
          static_cast<const __nv_bfloat16*>(d->L2), N, w->rank, 0, w->r_pad, w->l2t);
      if (cudaGetLastError() != cudaSuccess) {
        rc = SVDQ_ERR_CUDA;
        break;
      }
    }
    if ((rc = refold_l1(w, st))) break;
    if ((rc = quantize_residual(w, d->R, st))) break;
    if ((rc = copy_bias(w, d->bias, st))) break;
    if (cudaStreamSynchronize(st) != cudaSuccess) {
      rc = SVDQ_ERR_CUDA;
      break;
    }
    rc = encode_weight_maps(w);
  } while (false);
  if (rc) {
    free_weights(w);
    return rc;
  }
  *out = w;
  return SVDQ_OK;
}

SVDQ_API int svdq_append_lora(svdq_weights* w, const void* A, const void* B, int rl, void* stream) {
  if (w == nullptr || A == nullptr || B == nullptr || rl <= 0) return SVDQ_ERR_INVALID_ARG;
  int dev;
  int rc = current_device(&dev);
  if (rc) return rc;
  if (dev != w->device) return SVDQ_ERR_INVALID_ARG;
  return do_append_lora(w, A, B, rl, static_cast<cudaStream_t>(stream));
}

SVDQ_API int svdq_weights_scale_exponent(const svdq_weights* w, int* exponent) {
  if (w == nullptr || exponent == nullptr) return SVDQ_ERR_INVALID_ARG;
  *exponent = w->w_exp;
  return SVDQ_OK;
}

SVDQ_API int svdq_weights_refine_error(const svdq_weights* w, double* initial, double* kept) {
  if (w == nullptr) return SVDQ_ERR_INVALID_ARG;
  if (initial) *initial = w->refine_err0;
  if (kept) *kept = w->refine_err;
  return SVDQ_OK;
}

SVDQ_API int svdq_weights_info(const svdq_weights* w, int* fmt, int* K, int* N, int* rank,
                               int* rank_padded_out) {
  if (w == nullptr) return SVDQ_ERR_INVALID_ARG;
  if (fmt) *fmt = w->fmt;
  if (K) *K = w->K;
  if (N) *N = w->N;
  if (rank) *rank = w->rank;
  if (rank_padded_out) *rank_padded_out = w->r_pad;
  return SVDQ_OK;
}

SVDQ_API int svdq_act_workspace_bytes(const svdq_weights* w, int M, size_t* bytes) {
  if (w == nullptr || bytes == nullptr || M < 0) return SVDQ_ERR_INVALID_ARG;
  *bytes = act_layout(w, M).total;
  return SVDQ_OK;
}

SVDQ_API int svdq_quantize_act(const svdq_weights* w, const void* X, int M, void* ws, void* stream) {
  if (w == nullptr || M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (X == nullptr || ws == nullptr || !aligned16(X) || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return SVDQ_ERR_INVALID_ARG;
  int dev;
  int rc = current_device(&dev);
  if (rc) return rc;
  if (dev != w->device) return SVDQ_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const ActLayout L = act_layout(w, M);
  uint8_t* base = static_cast<uint8_t*>(ws);
  const QuantSplit sp = quant_split_for(w->fmt, M, w->K, w->r_pad, g_dev[dev]);
  const int S = sp.S;
  const int BM = kQuantTileRows / S;
  CUtensorMap tm_x, tm_codes;
  if ((rc = make_map(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, w->K, M, kQuantBK, BM)))
    return rc;
  // codes: NVFP4 M x K/2 packed E2M1, INT4 M x K int8; one box = a warp's
  // rows of one sub-tile, min(32, BM) rows
  const uint32_t rb = quant_code_row_bytes(w->fmt);
  if ((rc = make_map(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base + L.codes_off,
                     is_fp4(w->fmt) ? w->K / 2 : w->K, M, rb, std::min(BM, 32))))
    return rc;
  QuantParams p;
  p.M = M;
  p.K = w->K;
  p.r_pad = w->r_pad;
  p.S = S;
  p.C = sp.C;
  p.per = ((w->K + S * kQuantBK - 1) / (S * kQuantBK) + sp.C - 1) / sp.C;
  p.M_pad = L.M_pad;
  p.sf_kcols = w->sf_kcols;
  p.inv_lambda = w->inv_lambda;
  p.sf = base + L.sf_off;
  p.xl1 = reinterpret_cast<__nv_bfloat16*>(base + L.xl1_off);
  p.budget = wait_budget();
  const QuantSmem Q = quant_smem_layout(w->fmt, w->r_pad, S);
  if (Q.groups < 1 || Q.stages % Q.groups != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  // the X_hat L1 epilogue parks [128][r_pad + 4] fp32 over the stage and staging buffers
  if (static_cast<uint32_t>(kQuantTileRows * (w->r_pad + 4) * 4) > Q.bar_off) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (is_fp4(w->fmt) && w->sf_kcols * 64 != w->K) {
    // zero the scale atoms of the K padding (read by the GEMM's last K step)
    const size_t pitch = static_cast<size_t>(w->sf_kcols) * 512;
    const size_t off = static_cast<size_t>(w->K / 64) * 512;
    SVDQ_CUDA(cudaMemset2DAsync(p.sf + off, pitch, 0, pitch - off, L.M_pad / 128, st));
  }
  // clusters of C consecutive CTAs share a row block, one K range each
  const dim3 grid(((M + BM - 1) / BM) * sp.C);
  const unsigned C = static_cast<unsigned>(sp.C);
  const CUtensorMap& tm_l1t = w->r_pad > 0 ? w->tm_l1t : tm_x;
  const dim3 blk(kQuantThreads);
  if (w->fmt == SVDQ_NVFP4) {
    SVDQ_CUDA(launch_pdl(quant_act_kernel<0>, grid, blk, Q.total, st, C, tm_x, tm_l1t, tm_codes, p));
  } else if (w->fmt == SVDQ_FP4G32) {
    SVDQ_CUDA(launch_pdl(quant_act_kernel<2>, grid, blk, Q.total, st, C, tm_x, tm_l1t, tm_codes, p));
  } else if (w->fmt == SVDQ_W8A8) {
    // the per-token scales first: they need all of K before any code
    SVDQ_CUDA(launch_pdl(w8_row_scale_kernel, dim3((M + 7) / 8), dim3(256), 0, st, 0u,
                         static_cast<const __nv_bfloat16*>(X), static_cast<const float*>(w->inv_lambda), M,
                         w->K, reinterpret_cast<float*>(p.sf)));
    SVDQ_CUDA(launch_pdl(quant_act_kernel<3>, grid, blk, Q.total, st, C, tm_x, tm_l1t, tm_codes, p));
  } else {
    SVDQ_CUDA(launch_pdl(quant_act_kernel<1>, grid, blk, Q.total, st, C, tm_x, tm_l1t, tm_codes, p));
  }
  return SVDQ_OK;
}

// Row blocks per group of the GEMMs' tile order (gemm_tile_coords).
int gemm_group_m(int m_tiles, int n_tiles, int grid) {
  const int g = g_forced_group_m.load(std::memory_order_relaxed);
  if (g > 0) return std::min(g, m_tiles);
  (void)n_tiles;
  (void)grid;
  return std::min(kGemmGroupM, m_tiles);
}

// FP4 GEMM kernel: 1 = single CTAs (128 x 256 tiles), 2 = CTA pairs on
// 256 x 256 tiles, 3 = CTA pairs on 256 x 192 tiles with two accumulators.
// With one accumulator the MMAs of a tile wait until the epilogue has copied
// the previous tile out of TMEM; two accumulators hide that hand-off, which
// weighs most when the tiles are short in K.  On B200 the 192-column tiles are
// 3-5 % faster at K = 3072 (FLUX QKV, out and fc1 layers) and 6 % slower at
// K = 12288 (fc2), where a tile's K loop is four times longer.
int fp4_gemm_kind(const svdq_weights* w, const DeviceInfo& d) {
  const int forced = g_forced_gemm_kind.load(std::memory_order_relaxed);
  int kind = forced != 0 ? forced : (w->K <= 4096 ? 3 : 2);
  if (kind == 3 && d.pair192_clusters <= 0) kind = 2;
  if ((kind == 2 || kind == 4) && d.pair_clusters <= 0) kind = 1;
  return kind;
}

SVDQ_API int svdq_linear(const svdq_weights* w, const void* ws, int M, void* Y, void* stream) {
  if (w == nullptr || M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (ws == nullptr || Y == nullptr || !aligned16(Y) || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return SVDQ_ERR_INVALID_ARG;
  int dev;
  int rc = current_device(&dev);
  if (rc) return rc;
  if (dev != w->device) return SVDQ_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const ActLayout L = act_layout(w, M);
  const uint8_t* base = static_cast<const uint8_t*>(ws);
  CUtensorMap tm_a, tm_xl1;
  const int m_tiles = L.M_pad / 128;
  const int n_tiles = w->fmt != SVDQ_INT4 ? (w->N + kGemmBN - 1) / kGemmBN : (w->N + kI4BN - 1) / kI4BN;
  const int tiles = m_tiles * n_tiles;
  const int grid = std::min(tiles, g_dev[dev].sms);
  const int group_m = gemm_group_m(m_tiles, n_tiles, grid);
  if (is_fp4(w->fmt))
    rc = make_map(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base + L.codes_off, w->K / 2, M, 128, kGemmBM);
  else if (w->fmt == SVDQ_W8A8)
    rc = make_map(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base + L.codes_off, w->K, M, kW8BKB, kW8BM);
  else
    rc = make_map(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base + L.codes_off, w->K, M, 64, kI4BM);
  if (rc) return rc;
  if (w->r_pad > 0) {
    if ((rc = make_map(&tm_xl1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base + L.xl1_off, 2 * w->r_pad, M,
                       w->fmt != SVDQ_INT4 ? lr_chunk_cols(2 * w->r_pad) : i4_lr_chunk_cols(2 * w->r_pad),
                       128)))
      return rc;
  } else {
    tm_xl1 = tm_a;
  }
  const int fp4_kind = is_fp4(w->fmt) ? fp4_gemm_kind(w, g_dev[dev]) : 0;
  if (fp4_kind == 2 || fp4_kind == 3 || fp4_kind == 4) {
    const int bn = fp4_kind == 3 ? 192 : 256;
    CUtensorMap tm_y, tm_sfa;
    if ((rc = make_map(&tm_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Y, w->N, M, 32, 32))) return rc;
    if ((rc = make_atom_map(&tm_sfa, base + L.sf_off, static_cast<uint64_t>(L.M_pad / 128) * w->sf_kcols)))
      return rc;
    GemmParams p;
    p.M = M;
    p.N = w->N;
    p.K = w->K;
    p.kt_total = (w->K + 255) / 256;
    p.m_tiles = (M + kPairBM - 1) / kPairBM;
    p.n_tiles = (w->N + bn - 1) / bn;
    p.num_tiles = p.m_tiles * p.n_tiles;
    const int forced_g = g_forced_group_m.load(std::memory_order_relaxed);
    p.group_m = forced_g > 0 ? std::min((forced_g + 1) / 2, p.m_tiles) : std::min(kPairGroupM, p.m_tiles);
    // 256-column tiles left over after the last full round of the pairs, if at
    // most half as many as the pairs, go as two 256 x 128 units each
    const int pairs_max = bn == 256 ? g_dev[dev].pair_clusters : g_dev[dev].pair192_clusters;
    const int left = p.num_tiles % pairs_max;
    p.wide_tiles = (fp4_kind == 2 && left > 0 && 2 * left <= pairs_max) ? p.num_tiles - left : p.num_tiles;
    p.num_units = p.wide_tiles + 2 * (p.num_tiles - p.wide_tiles);
    p.r_tail = 2 * w->r_pad;
    p.sfa = nullptr;
    p.sfb = nullptr;
    p.sf_kcols = w->sf_kcols;
    p.bias = w->bias;
    p.out_scale = std::ldexp(1.0f, -w->w_exp);
    p.budget = wait_budget();
    if (bn == 256) {
      const int pairs = std::min(p.num_units, g_dev[dev].pair_clusters);
      SVDQ_CUDA(launch_pdl(gemm_nvfp4_pair_kernel<256>, dim3(2 * pairs), dim3(kGemmThreads), kPairSmemBytes, st,
                           2u, tm_a, w->tm_b_half, tm_sfa, w->tm_sfb, tm_xl1, w->tm_l2t_half, tm_y, p));
    } else {
      const int pairs = std::min(p.num_units, g_dev[dev].pair192_clusters);
      SVDQ_CUDA(launch_pdl(gemm_nvfp4_pair_kernel<192>, dim3(2 * pairs), dim3(kGemmThreads), kPair192SmemBytes,
                           st, 2u, tm_a, w->tm_b_96, tm_sfa, w->tm_sfb192, tm_xl1, w->tm_l2t_96, tm_y, p));
    }
  } else if (is_fp4(w->fmt)) {
    CUtensorMap tm_y;
    if ((rc = make_map(&tm_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Y, w->N, M, 16, 32))) return rc;
    GemmParams p;
    p.M = M;
    p.N = w->N;
    p.K = w->K;
    p.kt_total = (w->K + 255) / 256;
    p.m_tiles = m_tiles;
    p.n_tiles = n_tiles;
    p.num_tiles = tiles;
    p.group_m = group_m;
    p.wide_tiles = tiles;
    p.num_units = tiles;
    p.r_tail = 2 * w->r_pad;
    p.sfa = base + L.sf_off;
    p.sfb = w->wsf;
    p.sf_kcols = w->sf_kcols;
    p.bias = w->bias;
    p.out_scale = std::ldexp(1.0f, -w->w_exp);
    p.budget = wait_budget();
    SVDQ_CUDA(launch_pdl(gemm_nvfp4_kernel, dim3(grid), dim3(kGemmThreads), kGemmSmemBytes, st, 0u, tm_a,
                         w->tm_b, tm_xl1, w->tm_l2t, tm_y, p));
  } else if (w->fmt == SVDQ_W8A8) {
    CUtensorMap tm_y;
    if ((rc = make_map(&tm_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Y, w->N, M, 16, 32))) return rc;
    GemmW8Params p;
    p.M = M;
    p.N = w->N;
    p.K = w->K;
    p.kt_total = (w->K + kW8BKB - 1) / kW8BKB;
    p.m_tiles = m_tiles;
    p.n_tiles = n_tiles;
    p.num_tiles = tiles;
    p.group_m = group_m;
    p.r_tail = 2 * w->r_pad;
    p.sx = reinterpret_cast<const float*>(base + L.sf_off);
    p.sw = reinterpret_cast<const float*>(w->wsf);
    p.bias = w->bias;
    p.budget = wait_budget();
    SVDQ_CUDA(launch_pdl(gemm_w8a8_kernel, dim3(grid), dim3(kW8Threads), kW8SmemBytes, st, 0u, tm_a, w->tm_b,
                         tm_xl1, w->tm_l2t, tm_y, p));
  } else {
    GemmI4Params p;
    p.M = M;
    p.N = w->N;
    p.K = w->K;
    p.groups = w->K / 64;
    p.m_tiles = m_tiles;
    p.n_tiles = n_tiles;
    p.num_tiles = tiles;
    p.group_m = group_m;
    p.r_tail = 2 * w->r_pad;
    p.sx = reinterpret_cast<const uint16_t*>(base + L.sf_off);
    p.sw16 = w->wsw16;
    p.M_pad = L.M_pad;
    p.N_pad = w->N_pad;
    p.bias = w->bias;
    p.Y = static_cast<__nv_bfloat16*>(Y);
    p.budget = wait_budget();
    SVDQ_CUDA(launch_pdl(gemm_int4_kernel, dim3(grid), dim3(kI4Threads), kI4SmemBytes, st, 0u, tm_a, w->tm_b,
                         tm_xl1, w->tm_l2t, p));
  }
  SVDQ_CHECK_LAUNCH();
  return SVDQ_OK;
}

SVDQ_API int svdq_forward(const svdq_weights* w, const void* X, int M, void* Y, void* ws, void* stream) {
  int rc = svdq_quantize_act(w, X, M, ws, stream);
  if (rc) return rc;
  return svdq_linear(w, ws, M, Y, stream);
}

// ------------------------------------------------------------ no-allocation forward ---
// Some callers may not allocate device memory at all: a plugin inside a host
// framework that owns every device byte, or a latency-critical serving loop
// where cudaMalloc's implicit device-wide synchronization is not acceptable.
// svdq_forward_noalloc keeps the activation workspace in this fixed array
// instead.  Every GPU that loads the library holds it until the process exits.
static __device__ __align__(256) uint8_t g_noalloc_workspace[SVDQ_NOALLOC_WORKSPACE_BYTES];

SVDQ_API int svdq_forward_noalloc(const svdq_weights* w, const void* X, int M, void* Y, void* stream) {
  static std::atomic<void*> ws_ptr[kMaxDevices] = {};
  if (w == nullptr || M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  const size_t need = act_layout(w, M).total;
  if (need > SVDQ_NOALLOC_WORKSPACE_BYTES) {
    std::fprintf(stderr,
                 "svdq_forward_noalloc: M=%d K=%d rank_padded=%d needs a %zu-byte workspace, more than "
                 "the %u-byte fixed one; use svdq_forward with a caller workspace\n",
                 M, w->K, w->r_pad, need, static_cast<unsigned>(SVDQ_NOALLOC_WORKSPACE_BYTES));
    return SVDQ_ERR_UNSUPPORTED_SHAPE;
  }
  int dev;
  int rc = current_device(&dev);
  if (rc) return rc;
  if (dev != w->device) return SVDQ_ERR_INVALID_ARG;
  if (dev < 0 || dev >= kMaxDevices) return SVDQ_ERR_CUDA;   // (current_device checks this as well)
  void* ws = ws_ptr[dev].load(std::memory_order_acquire);
  if (ws == nullptr) {
    // first call on this device: look up the array's device address once
    // (host code cannot use the symbol itself as a device pointer)
    std::lock_guard<std::mutex> lk(g_mutex);
    ws = ws_ptr[dev].load(std::memory_order_relaxed);
    if (ws == nullptr) {
      const cudaError_t e = cudaGetSymbolAddress(&ws, g_noalloc_workspace);
      if (e != cudaSuccess) {
        std::fprintf(stderr, "svdq_forward_noalloc: cudaGetSymbolAddress failed: %s\n",
                     cudaGetErrorString(e));
        return SVDQ_ERR_CUDA;
      }
      ws_ptr[dev].store(ws, std::memory_order_release);
    }
  }
  // The activation kernel rewrites every workspace byte the GEMM reads for this
  // M (codes, scales including the K padding, XL1), so the array's previous
  // contents never leak into the result.
  return svdq_forward(w, X, M, Y, ws, stream);
}

SVDQ_API int svdq_export_act(const svdq_weights* w, const void* ws, int M, uint8_t* codes,
                             void* scales, void* xl1) {
  if (w == nullptr || ws == nullptr || M < 0) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  SVDQ_CUDA(cudaDeviceSynchronize());
  const ActLayout L = act_layout(w, M);
  const uint8_t* base = static_cast<const uint8_t*>(ws);
  const int K = w->K;
  if (codes) {
    if (is_fp4(w->fmt) || w->fmt == SVDQ_W8A8) {
      // packed E2M1 pairs, or W8A8's int8 codes as they are
      SVDQ_CUDA(cudaMemcpy(codes, base + L.codes_off, L.codes_bytes, cudaMemcpyDeviceToHost));
    } else {
      // INT4: int8 codes in the GEMM's K order (0 2 4 6 1 3 5 7 in each run of
      // eight) -> packed nibbles in natural order
      std::vector<int8_t> tmp(L.codes_bytes);
      SVDQ_CUDA(cudaMemcpy(tmp.data(), base + L.codes_off, L.codes_bytes, cudaMemcpyDeviceToHost));
      for (size_t c = 0; c < tmp.size() / 8; ++c) {
        const int8_t* e = tmp.data() + 8 * c;   // e[0..3] = k 0 2 4 6, e[4..7] = k 1 3 5 7
        for (int i = 0; i < 4; ++i)
          codes[4 * c + i] = static_cast<uint8_t>((e[i] & 0xF) | ((e[4 + i] & 0xF) << 4));
      }
    }
  }
  if (scales) {
    std::vector<uint8_t> tmp(L.sf_bytes);
    SVDQ_CUDA(cudaMemcpy(tmp.data(), base + L.sf_off, L.sf_bytes, cudaMemcpyDeviceToHost));
    if (is_fp4(w->fmt)) {
      // plain [M][K/g] from the atoms (FP4 g32: the first of each stored pair)
      uint8_t* out = static_cast<uint8_t*>(scales);
      const int step = w->fmt == SVDQ_FP4G32 ? 2 : 1;
      const int G = K / (16 * step);
      for (int m = 0; m < M; ++m)
        for (int g = 0; g < G; ++g) {
          const int b = g * step;   // block of 16
          const size_t atom = (static_cast<size_t>(m / 128) * w->sf_kcols + b / 4) * 512;
          out[static_cast<size_t>(m) * G + g] = tmp[atom + (m % 32) * 16 + ((m % 128) / 32) * 4 + b % 4];
        }
    } else if (w->fmt == SVDQ_W8A8) {
      std::memcpy(scales, tmp.data(), static_cast<size_t>(M) * 4);   // fp32 per token
    } else {
      uint16_t* out = static_cast<uint16_t*>(scales);
      const uint16_t* in = reinterpret_cast<const uint16_t*>(tmp.data());
      const int G = K / 64;
      for (int m = 0; m < M; ++m)
        for (int g = 0; g < G; ++g) out[static_cast<size_t>(m) * G + g] = in[static_cast<size_t>(g) * L.M_pad + m];
    }
  }
  if (xl1 && w->rank > 0) {
    // fp32 value = hi + lo (exact in fp32)
    std::vector<uint16_t> tmp(static_cast<size_t>(M) * 2 * w->r_pad);
    SVDQ_CUDA(cudaMemcpy(tmp.data(), base + L.xl1_off, tmp.size() * 2, cudaMemcpyDeviceToHost));
    float* out = static_cast<float*>(xl1);
    auto bf = [](uint16_t h) {
      const uint32_t u = static_cast<uint32_t>(h) << 16;
      float f;
      std::memcpy(&f, &u, 4);
      return f;
    };
    for (int m = 0; m < M; ++m)
      for (int j = 0; j < w->rank; ++j) {
        const size_t row = static_cast<size_t>(m) * 2 * w->r_pad;
        out[static_cast<size_t>(m) * w->rank + j] = bf(tmp[row + j]) + bf(tmp[row + w->r_pad + j]);
      }
  }
  return SVDQ_OK;
}

SVDQ_API int svdq_export_weights(const svdq_weights* w, uint8_t* codes, void* scales, void* L1,
                                 void* L2, float* inv_lambda, float* lambda) {
  if (w == nullptr) return SVDQ_ERR_INVALID_ARG;
  SVDQ_CUDA(cudaDeviceSynchronize());
  const int K = w->K, N = w->N;
  if (codes) {
    if (w->fmt == SVDQ_W8A8) {
      SVDQ_CUDA(cudaMemcpy(codes, w->wcodes, static_cast<size_t>(N) * K, cudaMemcpyDeviceToHost));
    } else {   // packed nibbles as stored (E2M1, or INT4 two's complement)
      SVDQ_CUDA(cudaMemcpy(codes, w->wcodes, static_cast<size_t>(N) * K / 2, cudaMemcpyDeviceToHost));
    }
  }
  if (scales) {
    if (is_fp4(w->fmt)) {
      const size_t bytes = static_cast<size_t>(w->N_pad / 128) * w->sf_kcols * 512;
      std::vector<uint8_t> tmp(bytes);
      SVDQ_CUDA(cudaMemcpy(tmp.data(), w->wsf, bytes, cudaMemcpyDeviceToHost));
      uint8_t* out = static_cast<uint8_t*>(scales);
      const int step = w->fmt == SVDQ_FP4G32 ? 2 : 1;
      const int G = K / (16 * step);
      for (int n = 0; n < N; ++n)
        for (int g = 0; g < G; ++g) {
          const int b = g * step;   // block of 16
          const size_t atom = (static_cast<size_t>(n / 128) * w->sf_kcols + b / 4) * 512;
          out[static_cast<size_t>(n) * G + g] = tmp[atom + (n % 32) * 16 + ((n % 128) / 32) * 4 + b % 4];
        }
    } else if (w->fmt == SVDQ_W8A8) {
      SVDQ_CUDA(cudaMemcpy(scales, w->wsf, static_cast<size_t>(N) * 4, cudaMemcpyDeviceToHost));
    } else {
      const int G = K / 64;
      std::vector<uint16_t> tmp(static_cast<size_t>(G) * w->N_pad);
      SVDQ_CUDA(cudaMemcpy(tmp.data(), w->wsf, tmp.size() * 2, cudaMemcpyDeviceToHost));
      uint16_t* out = static_cast<uint16_t*>(scales);
      for (int n = 0; n < N; ++n)
        for (int g = 0; g < G; ++g) out[static_cast<size_t>(n) * G + g] = tmp[static_cast<size_t>(g) * w->N_pad + n];
    }
  }
  if (L1 && w->rank > 0) {
    std::vector<uint16_t> tmp(static_cast<size_t>(w->r_pad) * K);
    SVDQ_CUDA(cudaMemcpy(tmp.data(), w->l1t, tmp.size() * 2, cudaMemcpyDeviceToHost));
    uint16_t* out = static_cast<uint16_t*>(L1);
    for (int k = 0; k < K; ++k)
      for (int j = 0; j < w->rank; ++j) out[static_cast<size_t>(k) * w->rank + j] = tmp[static_cast<size_t>(j) * K + k];
  }
  if (L2 && w->rank > 0) {
    std::vector<uint16_t> tmp(static_cast<size_t>(N) * w->r_pad);
    SVDQ_CUDA(cudaMemcpy(tmp.data(), w->l2t, tmp.size() * 2, cudaMemcpyDeviceToHost));
    uint16_t* out = static_cast<uint16_t*>(L2);
    for (int j = 0; j < w->rank; ++j)
      for (int n = 0; n < N; ++n) out[static_cast<size_t>(j) * N + n] = tmp[static_cast<size_t>(n) * w->r_pad + j];
  }
  if (inv_lambda) SVDQ_CUDA(cudaMemcpy(inv_lambda, w->inv_lambda, K * 4, cudaMemcpyDeviceToHost));
  if (lambda) SVDQ_CUDA(cudaMemcpy(lambda, w->lambda, K * 4, cudaMemcpyDeviceToHost));
  return SVDQ_OK;
}

SVDQ_API void svdq_weights_destroy(svdq_weights* w) { free_weights(w); }

}  // extern "C"
