// gemm_int4.cuh -- the INT4 (groups of 64, fp16 scales) variant of the fused
// 4-bit GEMM + low-rank up-projection + bias.
//
// SVDQuant Sec. 5.1: INT4 quantization uses groups of 64 with 16-bit scales.
// Per-group scales s_x[m,g] s_w[g,n] do not factor out of a K sum, so each
// 64-wide group is one tcgen05 kind::i8 product (two K=32 MMAs, codes held as
// int8) into one of four TMEM partial buffers; the drain warps scale every
// partial and accumulate it in fp32 registers while the tensor core fills the
// other buffers.  The low-rank tail (kind::f16, fp32) goes through the same
// buffers with scale 1.
//
// The integer partial P (|P| <= 64 * 49 < 2^22) reaches the drain already as
// fp32: each buffer is pre-filled with the bit pattern of 1.5 * 2^23 and the
// MMAs accumulate onto it, so the bits read back are those of 1.5 * 2^23 + P
// exactly, and one subtraction recovers P.  After reading a buffer the drain
// refills it.  The drain then costs three packed fp32x2 operations per two
// outputs (subtract, scale product, fused multiply-add).
//
//   warp 0    : TMA producer (A 128 x 64 int8, B 128 x 64 int8, the group's
//               activation scales (fp16) and weight scales (fp32); then the
//               XL1 / L2^T chunks of the low-rank tail)
//   warp 1    : TMEM owner, MMA issuer
//   warps 2-9 : drain + epilogue; warp w serves TMEM lane quarter w % 4 and
//               output columns [64 * ((w - 2) / 4), +64) of the 128 x 128 tile,
//               read from TMEM in two halves of 32 columns to stay within
//               168 registers (10 warps share four 16K-register sub-partitions).
#pragma once

#include "gemm_nvfp4.cuh"
#include "svdq_formats.cuh"
#include "svdq_ptx.cuh"

namespace svdq {

constexpr int kI4BM = 128;
constexpr int kI4BN = 128;
constexpr int kI4BK = 64;                 // one group
constexpr int kI4Threads = 320;
constexpr int kI4EpiWarps = 8;
constexpr int kI4Bufs = 4;                // TMEM partial buffers of kI4BN columns
constexpr uint32_t kI4AOff = 0;
constexpr uint32_t kI4BOff = kI4BM * 128;                  // 16384 (A region fits a 128 B-row tail chunk)
constexpr uint32_t kI4SxOff = kI4BOff + kI4BN * 128;       // 32768 (so does the B region)
constexpr uint32_t kI4SwOff = kI4SxOff + kI4BM * 2;        // 33024
constexpr uint32_t kI4StageBytes = 33792;                  // 33 KB, multiple of 1024
constexpr int kI4Stages = 6;
constexpr uint32_t kI4SmemBytes = kI4StageBytes * kI4Stages + 256 + 1024;
constexpr uint32_t kI4Magic = 0x4B400000u;                 // bits of 1.5 * 2^23
constexpr float kI4MagicF = 12582912.0f;

// Low-rank tail chunks of at most 64 bf16 columns (128-byte rows).
__host__ __device__ inline int i4_lr_chunk_cols(int k_tail) { return k_tail < 64 ? k_tail : 64; }
__host__ __device__ inline int i4_lr_num_chunks(int k_tail) {
  return k_tail == 0 ? 0 : (k_tail + 63) / 64;
}

struct GemmI4Params {
  int M, N, K;
  int groups;          // K / 64
  int m_tiles, n_tiles, num_tiles;
  int group_m;         // tile order (gemm_tile_coords)
  int r_tail;          // tail K: 2 r_pad (X_hat L1 as hi | lo against L2^T | L2^T), 0 = none
  const uint16_t* sx;  // fp16 [K/64][M_pad]
  const float* sw;     // fp32 [K/64][N_pad] (exact copies of the fp16 weight scales)
  int M_pad, N_pad;
  const __nv_bfloat16* bias;
  __nv_bfloat16* Y;
  long long budget;
};

__device__ __forceinline__ void tmem_st32_const(uint32_t taddr, uint32_t v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, "
      "%1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1};" ::"r"(taddr),
      "r"(v)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ unsigned long long f2_pack(float a, float b) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}

__device__ __forceinline__ unsigned long long u2_pack(uint32_t a, uint32_t b) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ float2 f2_unpack(unsigned long long v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}

// acc + s * (x - c), each lane of the pair rounded as sub, then fused multiply-add.
__device__ __forceinline__ unsigned long long f2_scale_acc(unsigned long long acc, unsigned long long x,
                                                           unsigned long long c, unsigned long long s) {
  unsigned long long p, r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(p) : "l"(x), "l"(c));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(p), "l"(s), "l"(acc));
  return r;
}

__device__ __forceinline__ unsigned long long f2_mul(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ unsigned long long f2_add(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__global__ void __launch_bounds__(kI4Threads, 1)
    gemm_int4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_xl1,
                     const __grid_constant__ CUtensorMap tm_l2t, const GemmI4Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  constexpr int S = kI4Stages;
  constexpr int NB = kI4Bufs;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kI4StageBytes * S);
  uint64_t* empty = full + S;
  uint64_t* pfull = empty + S;      // [NB]
  uint64_t* pempty = pfull + NB;    // [NB]
  uint64_t* mma_done = pempty + NB;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int n_lr = i4_lr_num_chunks(p.r_tail);
  const int lr_cols = i4_lr_chunk_cols(p.r_tail);
  const int steps_per_tile = p.groups + n_lr;

  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kI4EpiWarps);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(&pfull[b], 1);
      mbar_init(&pempty[b], kI4EpiWarps);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  if (warp >= 2) {
    // every partial buffer starts out holding the conversion offset
    const uint32_t q = warp & 3u, h = (warp - 2) >> 2;
    for (int b = 0; b < NB; ++b)
      for (int c = 0; c < 2; ++c)
        tmem_st32_const(tmem_base + ((q * 32u) << 16) + kI4BN * b + 64u * h + 32u * c, kI4Magic);
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();   // the activation codes, scales and XL1 come from the previous kernel

  if (warp == 0) {
    if (elect_one()) {
      prefetch_tmap(&tm_a);
      prefetch_tmap(&tm_b);
      if (n_lr) {
        prefetch_tmap(&tm_xl1);
        prefetch_tmap(&tm_l2t);
      }
      const uint32_t main_tx = kI4BM * 64 + kI4BN * 64 + kI4BM * 2 + kI4BN * 4;
      const uint32_t lr_tx = (kI4BM + kI4BN) * lr_cols * 2;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        int m_blk, n_blk;
        gemm_tile_coords(p.m_tiles, p.n_tiles, p.group_m, tile, m_blk, n_blk);
        const int m0 = m_blk * kI4BM, n0 = n_blk * kI4BN;
        for (int step = 0; step < steps_per_tile; ++step, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, p.budget, abort_flag)) {
            raise_error(kErrWaitGemm);
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kI4StageBytes;
          if (step < p.groups) {
            const int g = step;
            mbar_arrive_expect_tx(&full[s], main_tx);
            tma_load_2d(st + kI4AOff, &tm_a, &full[s], g * kI4BK, m0);
            tma_load_2d(st + kI4BOff, &tm_b, &full[s], g * kI4BK, n0);
            bulk_load(st + kI4SxOff, p.sx + static_cast<size_t>(g) * p.M_pad + m0, kI4BM * 2, &full[s]);
            bulk_load(st + kI4SwOff, p.sw + static_cast<size_t>(g) * p.N_pad + n0, kI4BN * 4, &full[s]);
          } else {
            const int c = step - p.groups;
            mbar_arrive_expect_tx(&full[s], lr_tx);
            tma_load_2d(st + kI4AOff, &tm_xl1, &full[s], c * 64, m0);
            tma_load_2d(st + kI4BOff, &tm_l2t, &full[s], c * 64, n0);
          }
        }
      }
      if (*abort_flag) {
        for (int i = (it > S ? it - S : 0); i < it; ++i)
          mbar_wait(&full[i % S], (i / S) & 1, p.budget, nullptr);
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      const uint32_t idesc_main = idesc_s8_s32(kI4BM, kI4BN);
      const uint32_t idesc_lr = idesc_bf16_f32(kI4BM, kI4BN);
      const uint32_t lr_row_bytes = static_cast<uint32_t>(lr_cols) * 2;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        for (int step = 0; step < steps_per_tile; ++step, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          const int b = it % NB;
          const uint32_t pph = (it / NB) & 1;
          const bool tail = step >= p.groups;
          if (!mbar_wait(&pempty[b], pph ^ 1, p.budget, abort_flag) ||
              !mbar_wait(&full[s], ph, p.budget, abort_flag)) {
            raise_error(kErrWaitGemm);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* st = smem + s * kI4StageBytes;
          const uint32_t a0 = smem_u32(st + kI4AOff), b0 = smem_u32(st + kI4BOff);
          const uint32_t d = tmem_base + kI4BN * b;
          if (!tail) {
            // accumulate onto the buffer's conversion offset
#pragma unroll
            for (int j = 0; j < 2; ++j)
              mma_i8(d, make_kmajor_desc(a0 + 32 * j, 64), make_kmajor_desc(b0 + 32 * j, 64),
                     idesc_main, 1u);
          } else {
            for (int j = 0; j < lr_cols / 16; ++j)
              mma_bf16(d, make_kmajor_desc(a0 + 32 * j, lr_row_bytes),
                       make_kmajor_desc(b0 + 32 * j, lr_row_bytes), idesc_lr, j > 0 ? 1u : 0u);
          }
          tc_commit(&empty[s]);
          tc_commit(&pfull[b]);
        }
      }
      tc_commit(mma_done);
    }
  } else {
    // ------------------------------------------------------------ drain / epilogue
    const uint32_t q = warp & 3u;
    const uint32_t h = (warp - 2) >> 2;
    const uint32_t row = q * 32 + lane;
    const unsigned long long magic2 = f2_pack(kI4MagicF, kI4MagicF);
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
      int m_blk, n_blk;
      gemm_tile_coords(p.m_tiles, p.n_tiles, p.group_m, tile, m_blk, n_blk);
      const int m = m_blk * kI4BM + static_cast<int>(row);
      unsigned long long acc[32];   // 64 fp32 accumulators, pairs of adjacent columns
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[j] = 0ull;
      for (int step = 0; step < steps_per_tile; ++step, ++it) {
        const int s = it % S;
        const int b = it % NB;
        const uint32_t pph = (it / NB) & 1;
        if (!warp_wait(&pfull[b], pph, p.budget, abort_flag)) {
          if (lane == 0) raise_error(kErrWaitGemm);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const bool main_step = step < p.groups;
        const uint8_t* st = smem + s * kI4StageBytes;
        const float sx = main_step
            ? __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(st + kI4SxOff)[row]))
            : 1.0f;
        const unsigned long long sx2 = f2_pack(sx, sx);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint32_t taddr = tmem_base + ((q * 32u) << 16) + kI4BN * b + 64u * h + 32u * c;
          uint32_t r[32];
          tmem_ld32(taddr, r);
          tmem_wait_ld();
          tmem_st32_const(taddr, kI4Magic);
          unsigned long long* a = acc + 16 * c;
          if (main_step) {
            const float4* swp = reinterpret_cast<const float4*>(st + kI4SwOff) + 16 * h + 8 * c;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 w = swp[j];
              a[2 * j] = f2_scale_acc(a[2 * j], u2_pack(r[4 * j], r[4 * j + 1]), magic2,
                                      f2_mul(sx2, f2_pack(w.x, w.y)));
              a[2 * j + 1] = f2_scale_acc(a[2 * j + 1], u2_pack(r[4 * j + 2], r[4 * j + 3]), magic2,
                                          f2_mul(sx2, f2_pack(w.z, w.w)));
            }
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) a[j] = f2_add(a[j], u2_pack(r[2 * j], r[2 * j + 1]));
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&pempty[b]);   // the buffer holds the offset again
          mbar_arrive(&empty[s]);    // done with this stage's scales
        }
      }
      if (!ok) break;
      // bias, bf16, store
      const int n_base = n_blk * kI4BN + 64 * static_cast<int>(h);
      if (m < p.M) {
        __nv_bfloat16* yrow = p.Y + static_cast<size_t>(m) * p.N;
#pragma unroll
        for (int j = 0; j < 64; j += 8) {
          const int n = n_base + j;
          if (n < p.N) {
            float bb[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (p.bias != nullptr) {
              const uint4 w = __ldg(reinterpret_cast<const uint4*>(p.bias + n));
              const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                bb[2 * t] = bf16_lo(w4[t]);
                bb[2 * t + 1] = bf16_hi(w4[t]);
              }
            }
            float v[8];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const float2 a = f2_unpack(acc[j / 2 + t]);
              v[2 * t] = a.x + bb[2 * t];
              v[2 * t + 1] = a.y + bb[2 * t + 1];
            }
            uint4 o;
            o.x = pack_bf16x2(v[0], v[1]);
            o.y = pack_bf16x2(v[2], v[3]);
            o.z = pack_bf16x2(v[4], v[5]);
            o.w = pack_bf16x2(v[6], v[7]);
            *reinterpret_cast<uint4*>(yrow + n) = o;
          }
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    mbar_wait(mma_done, 0, p.budget, nullptr);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace svdq
