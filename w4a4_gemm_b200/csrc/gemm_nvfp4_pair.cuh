// gemm_nvfp4_pair.cuh -- the fused 4-bit GEMM on CTA pairs (256 x 256 tiles).
//
// Computes what gemm_nvfp4_kernel computes (SVDQuant Sec. 4.2, Eq. 5 and the
// fused low-rank branch of Sec. 4.3, Fig. 6b):
//   Y = Q(X_hat) Q(R) + (X_hat L1) L2 + b
// with every output tile shared by the two CTAs of a cluster.  The pair's
// 256 x 256 tile is one tcgen05.mma.cta_group::2 of M = 256, N = 256 per 64
// values of K: each CTA stages its own 128 activation rows and one half (128
// weight columns) of B, and the MMA, issued by rank 0, reads both CTAs'
// operands and accumulates each CTA's 128 x 256 block in that CTA's TMEM.
// Against one CTA per 128 x 256 tile, an SM then pulls 32 KB of codes per
// 256-wide K step instead of 48 KB for the same tensor-core work, and the
// smaller stages fit five to a CTA instead of four.
//
// Per CTA of the pair:
//   warp 0    : TMA producer for this CTA's stage buffers: A codes (128 x 128 B),
//               its half of B (128 x 128 B), the A scale atoms of its rows and
//               the B scale atoms of all 256 columns (every CTA's TMEM needs
//               them), then the low-rank operands (its XL1 rows, its half of
//               [L2^T | L2^T]).  All of them count on rank 0's stage barrier;
//               rank 0 alone arms it with both CTAs' bytes.
//   warp 1    : TMEM (allocated for the pair); on rank 0 one lane moves both
//               CTAs' scales into their TMEM (tcgen05.cp.cta_group::2) and
//               issues the pair MMAs; each commit signals the matching barrier
//               in both CTAs.
//   warps 2-9 : epilogue of this CTA's 128 rows, as in gemm_nvfp4_kernel; the
//               hand-back of the accumulator counts on rank 0's barrier, which
//               waits for all sixteen epilogue warps of the pair.
#pragma once

#include "gemm_nvfp4.cuh"

namespace svdq {

constexpr int kPairBM = 256;                   // rows per pair tile (128 per CTA)
constexpr int kPairBN = 256;                   // weight columns per pair tile (128 per CTA)
constexpr int kPairStages = 5;
constexpr int kPairGroupM = 4;                 // pair row blocks per tile-order group
constexpr uint32_t kPairAOff = 0;                                 // 128 x 128 B
constexpr uint32_t kPairBOff = 128 * kGemmBKB;                    // 16384: 128 x 128 B
constexpr uint32_t kPairSfaOff = kPairBOff + 128 * kGemmBKB;      // 32768: 4 atoms
constexpr uint32_t kPairSfbOff = kPairSfaOff + 4 * 512;           // 34816: 2 x 4 atoms
constexpr uint32_t kPairStageBytes = kPairSfbOff + 8 * 512;       // 38912 (38 x 1024)
constexpr uint32_t kPairEpiOff = kPairStageBytes * kPairStages;
constexpr uint32_t kPairBarOff = kPairEpiOff + kGemmEpiWarps * kGemmEpiBufBytes;
constexpr uint32_t kPairSmemBytes = kPairBarOff + 256 + 1024;
constexpr uint16_t kPairMask = 3;              // both CTAs of the pair

// p.m_tiles counts pair row blocks (256 rows); p.sfa / p.sfb are unused (the
// scale atoms come through tm_sfa / tm_sfb: [atoms][128 x 32-bit words]).
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_nvfp4_pair_kernel(const __grid_constant__ CUtensorMap tm_a,
                           const __grid_constant__ CUtensorMap tm_b,
                           const __grid_constant__ CUtensorMap tm_sfa,
                           const __grid_constant__ CUtensorMap tm_sfb,
                           const __grid_constant__ CUtensorMap tm_xl1,
                           const __grid_constant__ CUtensorMap tm_l2t,
                           const __grid_constant__ CUtensorMap tm_y, const GemmParams p) {
  constexpr int STAGES = kPairStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kPairBarOff);   // rank 0's are used
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 1;                                  // rank 0's is used
  uint64_t* mma_done = acc_empty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const uint32_t rank = cluster_ctarank();
  const int n_lr = lr_num_chunks(p.r_tail);
  const int lr_cols = lr_chunk_cols(p.r_tail);
  const int steps_per_tile = p.kt_total + n_lr;
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int n_pairs = static_cast<int>(gridDim.x >> 1);

  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * kGemmEpiWarps);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, kGemmTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // both CTAs' barriers and TMEM exist before either signals the other
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  griddep_wait();   // the activation codes, scales and XL1 come from the previous kernel

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (elect_one()) {
      prefetch_tmap(&tm_a);
      prefetch_tmap(&tm_b);
      prefetch_tmap(&tm_sfa);
      prefetch_tmap(&tm_sfb);
      if (n_lr) {
        prefetch_tmap(&tm_xl1);
        prefetch_tmap(&tm_l2t);
      }
      const uint32_t full0 = map_shared_rank(smem_u32(&full[0]), 0);   // rank 0's stage barriers
      const uint32_t main_tx = 2 * kPairStageBytes;
      const uint32_t lr_tx = 2 * 2 * 128 * static_cast<uint32_t>(lr_cols) * 2;
      int it = 0;
      bool ok = true;
      for (int tile = pair; tile < p.num_tiles && ok; tile += n_pairs) {
        int mp, nb;
        gemm_tile_coords(p.m_tiles, p.n_tiles, p.group_m, tile, mp, nb);
        const int m_blk = 2 * mp + static_cast<int>(rank);    // this CTA's 128-row block
        const int m0 = m_blk * 128;
        const int nh0 = nb * kPairBN + 128 * static_cast<int>(rank);
        for (int step = 0; step < steps_per_tile; ++step, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, p.budget, abort_flag)) {
            raise_error(kErrWaitGemm);
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kPairStageBytes;
          const uint32_t fb = full0 + static_cast<uint32_t>(s) * 8u;
          if (step < p.kt_total) {
            const int kt = step;
            if (rank == 0) mbar_arrive_expect_tx(&full[s], main_tx);
            tma_load_2d_pair(st + kPairAOff, &tm_a, fb, kt * kGemmBKB, m0);
            tma_load_2d_pair(st + kPairBOff, &tm_b, fb, kt * kGemmBKB, nh0);
            tma_load_2d_pair(st + kPairSfaOff, &tm_sfa, fb, 0, m_blk * p.sf_kcols + 4 * kt);
            tma_load_2d_pair(st + kPairSfbOff, &tm_sfb, fb, 0, (2 * nb) * p.sf_kcols + 4 * kt);
            tma_load_2d_pair(st + kPairSfbOff + 2048, &tm_sfb, fb, 0, (2 * nb + 1) * p.sf_kcols + 4 * kt);
          } else {
            const int c = step - p.kt_total;
            if (rank == 0) mbar_arrive_expect_tx(&full[s], lr_tx);
            tma_load_2d_pair(st + kPairAOff, &tm_xl1, fb, c * 64, m0);
            tma_load_2d_pair(st + kPairBOff, &tm_l2t, fb, c * 64, nh0);
          }
        }
      }
      if (*abort_flag && rank == 0) {
        for (int i = (it > STAGES ? it - STAGES : 0); i < it; ++i)
          mbar_wait(&full[i % STAGES], (i / STAGES) & 1, p.budget, nullptr);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (rank 0)
    if (rank == 0 && elect_one()) {
      const uint32_t idesc_main = idesc_e2m1_ue4m3(kPairBM, kPairBN);
      const uint32_t idesc_lr = idesc_bf16_f32(kPairBM, kPairBN);
      const uint32_t lr_row_bytes = static_cast<uint32_t>(lr_cols) * 2;
      const uint32_t d_tmem = tmem_base;
      int it = 0, t_local = 0;
      bool ok = true;
      for (int tile = pair; tile < p.num_tiles && ok; tile += n_pairs, ++t_local) {
        if (!mbar_wait(acc_empty, (t_local & 1) ^ 1, p.budget, abort_flag)) {
          raise_error(kErrWaitGemm);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        for (int step = 0; step < steps_per_tile; ++step, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          const bool tail = step >= p.kt_total;
          if (!mbar_wait(&full[s], ph, p.budget, abort_flag)) {
            raise_error(kErrWaitGemm);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* st = smem + s * kPairStageBytes;
          const uint32_t a0 = smem_u32(st + kPairAOff);
          const uint32_t b0 = smem_u32(st + kPairBOff);
          if (!tail) {
            const uint32_t sfa_s = smem_u32(st + kPairSfaOff);
            const uint32_t sfb_s = smem_u32(st + kPairSfbOff);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              tmem_cp_32x128b_x4_pair(tmem_base + kGemmSfaCol + 4 * j, sf_desc(sfa_s + 512 * j));
              tmem_cp_32x128b_x4_pair(tmem_base + kGemmSfbCol + 8 * j, sf_desc(sfb_s + 512 * j));
              tmem_cp_32x128b_x4_pair(tmem_base + kGemmSfbCol + 8 * j + 4, sf_desc(sfb_s + 2048 + 512 * j));
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              mma_nvf4_pair(d_tmem, make_kmajor_desc(a0 + 32 * j, 128), make_kmajor_desc(b0 + 32 * j, 128),
                            idesc_main, tmem_base + kGemmSfaCol + 4 * j, tmem_base + kGemmSfbCol + 8 * j,
                            (step > 0 || j > 0) ? 1u : 0u);
            }
          } else {
            for (int j = 0; j < lr_cols / 16; ++j) {
              mma_bf16_pair(d_tmem, make_kmajor_desc(a0 + 32 * j, lr_row_bytes),
                            make_kmajor_desc(b0 + 32 * j, lr_row_bytes), idesc_lr, 1u);
            }
          }
          tc_commit_pair(&empty[s], kPairMask);
        }
        if (!ok) break;
        tc_commit_pair(acc_full, kPairMask);
      }
      tc_commit_pair(mma_done, kPairMask);   // retires once every MMA and copy issued above has completed
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const uint32_t q = warp & 3u;
    const uint32_t h = (warp - 2) >> 2;
    uint8_t* ebuf = smem + kPairEpiOff + (warp - 2) * kGemmEpiBufBytes;
    const uint32_t acc_empty0 = map_shared_rank(smem_u32(acc_empty), 0);
    int t_local = 0;
    for (int tile = pair; tile < p.num_tiles; tile += n_pairs, ++t_local) {
      int mp, nb;
      gemm_tile_coords(p.m_tiles, p.n_tiles, p.group_m, tile, mp, nb);
      if (!warp_wait(acc_full, t_local & 1, p.budget, abort_flag)) {
        if (lane == 0) raise_error(kErrWaitGemm);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      uint32_t v[4][32];
      const uint32_t taddr = tmem_base + ((q * 32u) << 16) + 128u * h;
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(taddr + 32 * c, v[c]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0);
      const int row0 = mp * kPairBM + 128 * static_cast<int>(rank) + static_cast<int>(q) * 32;
      const int ncol = nb * kPairBN + 128 * static_cast<int>(h);
      if (row0 < p.M) {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (ncol + 16 * c < p.N)
            epi_store_16(&v[c / 2][16 * (c % 2)], ebuf, &tm_y, ncol + 16 * c, row0, p.N, p.bias,
                         p.out_scale, lane);
      }
    }
    if (lane == 0) bulk_wait_group_all();
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // every MMA of the pair has retired before its TMEM is released
    mbar_wait(mma_done, 0, p.budget, nullptr);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kGemmTmemCols);
  }
  // neither CTA leaves while the other may still signal its barriers or read
  // its shared memory
  cluster_sync();
}

}  // namespace svdq
