// gemm_w8a8.cuh -- the 8-bit variant of the fused GEMM + low-rank up-projection.
//
// SVDQuant paper, Sec. 5.1 (8-bit setting): int8 activations with one scale
// per token row (computed at run time), int8 weights with one scale per
// output channel, and the 16-bit low-rank branch.  The scales are constant
// along K, so the whole K sum runs on the tensor core in int32 (exact:
// |sum| < 127^2 K < 2^31) and is scaled once in the epilogue:
//   y = bf16( fp32(acc) * (s_x[m] s_w[n]) + (X_hat L1) L2 + b )
// The low-rank tail (kind::f16, fp32) needs its own TMEM accumulator: columns
// 0..255 hold the int32 sum, 256..511 the fp32 tail.
//
//   warp 0    : TMA producer.  Per 128-wide K step: A codes (128 x 128 B int8),
//               B codes (256 x 128 B); then the low-rank operands XL1 (hi | lo)
//               and [L2^T | L2^T] in chunks of 64 columns.
//   warp 1    : TMEM owner, MMA issuer (kind::i8 into the int32 accumulator,
//               kind::f16 into the tail accumulator).
//   warps 2-9 : epilogue; warp w serves TMEM lane quarter w % 4 and columns
//               [128 h, 128 h + 128), h = (w - 2) / 4, in chunks of 32: both
//               accumulators -> registers, scale, add, bias, bf16, staged TMA
//               stores.  The TMEM goes back after the last chunk is read.
#pragma once

#include "gemm_nvfp4.cuh"
#include "svdq_formats.cuh"
#include "svdq_ptx.cuh"

namespace svdq {

constexpr int kW8BM = 128;
constexpr int kW8BN = 256;
constexpr int kW8BKB = 128;                    // K step: 128 int8 values
constexpr int kW8Threads = 320;
constexpr int kW8EpiWarps = 8;
constexpr uint32_t kW8LrCol = 256;             // fp32 tail accumulator
constexpr uint32_t kW8AOff = 0;
constexpr uint32_t kW8BOff = kW8BM * kW8BKB;                        // 16384
constexpr uint32_t kW8StageBytes = kW8BOff + kW8BN * kW8BKB;        // 49152
constexpr int kW8Stages = 4;
constexpr uint32_t kW8EpiOff = kW8StageBytes * kW8Stages;
constexpr uint32_t kW8BarOff = kW8EpiOff + kW8EpiWarps * kGemmEpiBufBytes;
constexpr uint32_t kW8SmemBytes = kW8BarOff + 256 + 1024;

struct GemmW8Params {
  int M, N, K;
  int kt_total;        // ceil(K / 128)
  int m_tiles, n_tiles, num_tiles;
  int group_m;         // tile order (gemm_tile_coords)
  int r_tail;          // 2 r_pad, 0 = no low-rank branch
  const float* sx;     // M_pad per-token scales
  const float* sw;     // N_pad per-channel scales
  const __nv_bfloat16* bias;
  long long budget;
};

__global__ void __launch_bounds__(kW8Threads, 1)
    gemm_w8a8_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_xl1,
                     const __grid_constant__ CUtensorMap tm_l2t,
                     const __grid_constant__ CUtensorMap tm_y, const GemmW8Params p) {
  constexpr int STAGES = kW8Stages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kW8BarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* mma_done = acc_empty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int n_lr = lr_num_chunks(p.r_tail);
  const int lr_cols = lr_chunk_cols(p.r_tail);
  const int steps_per_tile = p.kt_total + n_lr;

  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kW8EpiWarps);
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
  griddep_wait();   // the activation codes, scales and XL1 come from the previous kernel

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (elect_one()) {
      prefetch_tmap(&tm_a);
      prefetch_tmap(&tm_b);
      if (n_lr) {
        prefetch_tmap(&tm_xl1);
        prefetch_tmap(&tm_l2t);
      }
      const uint32_t lr_tx = (kW8BM + kW8BN) * lr_cols * 2;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        int m_blk, n_blk;
        gemm_tile_coords(p.m_tiles, p.n_tiles, p.group_m, tile, m_blk, n_blk);
        const int m0 = m_blk * kW8BM, n0 = n_blk * kW8BN;
        for (int step = 0; step < steps_per_tile; ++step, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, p.budget, abort_flag)) {
            raise_error(kErrWaitGemm);
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kW8StageBytes;
          if (step < p.kt_total) {
            mbar_arrive_expect_tx(&full[s], kW8StageBytes);
            tma_load_2d(st + kW8AOff, &tm_a, &full[s], step * kW8BKB, m0);
            tma_load_2d(st + kW8BOff, &tm_b, &full[s], step * kW8BKB, n0);
          } else {
            const int c = step - p.kt_total;
            mbar_arrive_expect_tx(&full[s], lr_tx);
            tma_load_2d(st + kW8AOff, &tm_xl1, &full[s], c * 64, m0);
            tma_load_2d(st + kW8BOff, &tm_l2t, &full[s], c * 64, n0);
          }
        }
      }
      // never leave while a copy into this CTA's shared memory is still in flight
      // (whether or not a wait ran out, and in whichever role)
      for (int i = (it > STAGES ? it - STAGES : 0); i < it; ++i)
        mbar_wait(&full[i % STAGES], (i / STAGES) & 1, drain_budget(p.budget), nullptr);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (elect_one()) {
      const uint32_t idesc_main = idesc_s8_s32(kW8BM, kW8BN);
      const uint32_t idesc_lr = idesc_bf16_f32(kW8BM, kW8BN);
      const uint32_t lr_row_bytes = static_cast<uint32_t>(lr_cols) * 2;
      int it = 0, t_local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++t_local) {
        if (!mbar_wait(acc_empty, (t_local & 1) ^ 1, p.budget, abort_flag)) {
          raise_error(kErrWaitGemm);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        for (int step = 0; step < steps_per_tile; ++step, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&full[s], ph, p.budget, abort_flag)) {
            raise_error(kErrWaitGemm);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* st = smem + s * kW8StageBytes;
          const uint32_t a0 = smem_u32(st + kW8AOff);
          const uint32_t b0 = smem_u32(st + kW8BOff);
          if (step < p.kt_total) {
#pragma unroll
            for (int j = 0; j < 4; ++j)   // K = 32 int8 per MMA
              mma_i8(tmem_base, make_kmajor_desc(a0 + 32 * j, 128), make_kmajor_desc(b0 + 32 * j, 128),
                     idesc_main, (step > 0 || j > 0) ? 1u : 0u);
          } else {
            const int c = step - p.kt_total;
            for (int j = 0; j < lr_cols / 16; ++j)
              mma_bf16(tmem_base + kW8LrCol, make_kmajor_desc(a0 + 32 * j, lr_row_bytes),
                       make_kmajor_desc(b0 + 32 * j, lr_row_bytes), idesc_lr, (c > 0 || j > 0) ? 1u : 0u);
          }
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
      tc_commit(mma_done);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const uint32_t q = warp & 3u;
    const uint32_t h = (warp - 2) >> 2;
    uint8_t* ebuf = smem + kW8EpiOff + (warp - 2) * kGemmEpiBufBytes;
    const bool has_lr = n_lr > 0;
    int t_local = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++t_local) {
      int m_blk, n_blk;
      gemm_tile_coords(p.m_tiles, p.n_tiles, p.group_m, tile, m_blk, n_blk);
      if (!warp_wait(acc_full, t_local & 1, p.budget, abort_flag)) {
        if (lane == 0) raise_error(kErrWaitGemm);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int row0 = m_blk * kW8BM + static_cast<int>(q) * 32;
      const int m = row0 + static_cast<int>(lane);
      const float sx = m < p.M ? p.sx[m] : 0.0f;
      const int nb = n_blk * kW8BN + 128 * static_cast<int>(h);
      const uint32_t taddr = tmem_base + ((q * 32u) << 16) + 128u * h;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t acc[32], lr[32];
        tmem_ld32(taddr + 32 * c, acc);
        if (has_lr) tmem_ld32(taddr + kW8LrCol + 32 * c, lr);
        tmem_wait_ld();
        if (c == 3) {   // both accumulators are in registers: hand the TMEM back
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(acc_empty);
        }
        const int n0 = nb + 32 * c;
        uint32_t y[32];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          float4 sw = make_float4(0.f, 0.f, 0.f, 0.f);
          if (n0 + e < p.N) sw = __ldg(reinterpret_cast<const float4*>(p.sw + n0 + e));
          const float s4[4] = {sw.x, sw.y, sw.z, sw.w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float a = __int2float_rn(static_cast<int>(acc[e + t]));
            y[e + t] = __float_as_uint(fmaf(a, sx * s4[t], has_lr ? __uint_as_float(lr[e + t]) : 0.0f));
          }
        }
        if (row0 < p.M) {
          if (n0 < p.N) epi_store_16(y, ebuf, &tm_y, n0, row0, p.N, p.bias, 1.0f, lane);
          if (n0 + 16 < p.N) epi_store_16(y + 16, ebuf, &tm_y, n0 + 16, row0, p.N, p.bias, 1.0f, lane);
        }
      }
    }
    if (lane == 0) bulk_wait_group_all();
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    mbar_wait(mma_done, 0, drain_budget(p.budget), nullptr);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace svdq
