// gemm_int4.cuh -- the INT4 (groups of 64, fp16 scales) variant of the fused
// 4-bit GEMM + low-rank up-projection + bias.
//
// SVDQuant Sec. 5.1: INT4 quantization uses groups of 64 with 16-bit scales.
// Per-group scales s_x[m,g] s_w[g,n] do not factor out of a K sum, so each
// 64-wide group is one tcgen05 kind::i8 product (two K=32 MMAs, codes held as
// int8) into one of two TMEM partial buffers; the epilogue warps drain every
// partial, scale it and accumulate it in fp32 registers while the tensor core
// fills the other buffer.  The low-rank tail (kind::f16, fp32) goes through
// the same buffers with scale 1.
//
//   warp 0    : TMA producer (A 128 x 64 int8, B 256 x 64 int8, the group's
//               activation and weight scales; then XL1 / L2^T chunks)
//   warp 1    : TMEM owner, MMA issuer
//   warps 2-9 : epilogue; warp w drains TMEM lane quarter w % 4 and output
//               columns [128 * ((w - 2) / 4), +128) of the 128 x 256 tile.
#pragma once

#include "gemm_nvfp4.cuh"
#include "svdq_formats.cuh"
#include "svdq_ptx.cuh"

namespace svdq {

constexpr int kI4BM = 128;
constexpr int kI4BN = 256;
constexpr int kI4BK = 64;                 // one group
constexpr int kI4Threads = 320;
constexpr int kI4EpiWarps = 8;
constexpr uint32_t kI4AOff = 0;
constexpr uint32_t kI4BOff = kI4BM * 128;                  // 16384 (A region fits a 128 B-row tail chunk)
constexpr uint32_t kI4SxOff = kI4BOff + kI4BN * 128;       // 49152 (so does the B region)
constexpr uint32_t kI4SwOff = kI4SxOff + kI4BM * 2;        // 49408
constexpr uint32_t kI4StageBytes = 50176;                  // 49 KB, multiple of 1024
constexpr int kI4Stages = 4;
constexpr uint32_t kI4SmemBytes = kI4StageBytes * kI4Stages + 256 + 1024;

struct GemmI4Params {
  int M, N, K;
  int groups;          // K / 64
  int m_tiles, n_tiles, num_tiles;
  int r_tail;          // tail K: 2 r_pad (X_hat L1 as hi | lo against L2^T | L2^T), 0 = none
  const uint16_t* sx;  // fp16 [K/64][M_pad]
  const uint16_t* sw;  // fp16 [K/64][N_pad]
  int M_pad, N_pad;
  const __nv_bfloat16* bias;
  __nv_bfloat16* Y;
  long long budget;
};

__global__ void __launch_bounds__(kI4Threads, 1)
    gemm_int4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_xl1,
                     const __grid_constant__ CUtensorMap tm_l2t, const GemmI4Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  constexpr int S = kI4Stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kI4StageBytes * S);
  uint64_t* empty = full + S;
  uint64_t* pfull = empty + S;      // [2]
  uint64_t* pempty = pfull + 2;     // [2]
  uint64_t* mma_done = pempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int n_lr = lr_num_chunks(p.r_tail);
  const int lr_cols = lr_chunk_cols(p.r_tail);
  const int steps_per_tile = p.groups + n_lr;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kI4EpiWarps);
    }
    for (int b = 0; b < 2; ++b) {
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

  if (warp == 0) {
    if (elect_one()) {
      prefetch_tmap(&tm_a);
      prefetch_tmap(&tm_b);
      if (n_lr) {
        prefetch_tmap(&tm_xl1);
        prefetch_tmap(&tm_l2t);
      }
      const uint32_t main_tx = kI4BM * 64 + kI4BN * 64 + kI4BM * 2 + kI4BN * 2;
      const uint32_t lr_tx = (kI4BM + kI4BN) * lr_cols * 2;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        const int m_blk = tile % p.m_tiles, n_blk = tile / p.m_tiles;
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
            bulk_load(st + kI4SwOff, p.sw + static_cast<size_t>(g) * p.N_pad + n0, kI4BN * 2, &full[s]);
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
          const int b = it & 1;
          const uint32_t pph = (it >> 1) & 1;
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
          const uint32_t d = tmem_base + 256u * b;
          if (!tail) {
#pragma unroll
            for (int j = 0; j < 2; ++j)
              mma_i8(d, make_kmajor_desc(a0 + 32 * j, 64), make_kmajor_desc(b0 + 32 * j, 64),
                     idesc_main, j > 0 ? 1u : 0u);
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
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
      const int m_blk = tile % p.m_tiles, n_blk = tile / p.m_tiles;
      const int m = m_blk * kI4BM + static_cast<int>(row);
      float acc[128];
#pragma unroll
      for (int j = 0; j < 128; ++j) acc[j] = 0.f;
      for (int step = 0; step < steps_per_tile; ++step, ++it) {
        const int s = it % S;
        const int b = it & 1;
        const uint32_t pph = (it >> 1) & 1;
        if (!warp_wait(&pfull[b], pph, p.budget, abort_flag)) {
          if (lane == 0) raise_error(kErrWaitGemm);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* st = smem + s * kI4StageBytes;
        const bool main_step = step < p.groups;
        const float sx = main_step
            ? __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(st + kI4SxOff)[row]))
            : 1.0f;
        const uint16_t* swp = reinterpret_cast<const uint16_t*>(st + kI4SwOff) + 128 * h;
        const uint32_t taddr = tmem_base + 256u * b + ((q * 32u) << 16) + 128u * h;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(taddr + 32 * c, r);
          tmem_wait_ld();
          if (main_step) {
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              const uint4 w = *reinterpret_cast<const uint4*>(swp + 32 * c + j);
              const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                const float2 s2 = __half22float2(*reinterpret_cast<const __half2*>(&w4[t]));
                // exact int32 -> fp32 for |P| < 2^22: add the bits of 1.5 * 2^23, subtract
                const float p0 = __int_as_float(static_cast<int>(r[j + 2 * t]) + 0x4B400000) - 12582912.0f;
                const float p1 = __int_as_float(static_cast<int>(r[j + 2 * t + 1]) + 0x4B400000) - 12582912.0f;
                acc[32 * c + j + 2 * t] = fmaf(sx * s2.x, p0, acc[32 * c + j + 2 * t]);
                acc[32 * c + j + 2 * t + 1] = fmaf(sx * s2.y, p1, acc[32 * c + j + 2 * t + 1]);
              }
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[32 * c + j] += __uint_as_float(r[j]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&pempty[b]);
          mbar_arrive(&empty[s]);
        }
      }
      if (!ok) break;
      // bias, bf16, store
      const int n_base = n_blk * kI4BN + 128 * static_cast<int>(h);
      if (m < p.M) {
        __nv_bfloat16* yrow = p.Y + static_cast<size_t>(m) * p.N;
#pragma unroll
        for (int j = 0; j < 128; j += 8) {
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
            uint4 o;
            o.x = pack_bf16x2(acc[j + 0] + bb[0], acc[j + 1] + bb[1]);
            o.y = pack_bf16x2(acc[j + 2] + bb[2], acc[j + 3] + bb[3]);
            o.z = pack_bf16x2(acc[j + 4] + bb[4], acc[j + 5] + bb[5]);
            o.w = pack_bf16x2(acc[j + 6] + bb[6], acc[j + 7] + bb[7]);
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
