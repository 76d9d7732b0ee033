// gemm_nvfp4_pair.cuh -- the fused 4-bit GEMM on CTA pairs (256 x BN tiles,
// BN = 256 or 192).
//
// Computes what gemm_nvfp4_kernel computes (SVDQuant Sec. 4.2, Eq. 5 and the
// fused low-rank branch of Sec. 4.3, Fig. 6b):
//   Y = Q(X_hat) Q(R) + (X_hat L1) L2 + b
// with every output tile shared by the two CTAs of a cluster.  The pair's
// 256 x BN tile is one tcgen05.mma.cta_group::2 of M = 256, N = BN per 64
// values of K: each CTA stages its own 128 activation rows and one half (BN / 2
// weight columns) of B, and the MMA, issued by rank 0, reads both CTAs'
// operands and accumulates each CTA's 128 x BN block in that CTA's TMEM.
// Against one CTA per 128 x 256 tile, an SM then pulls 32 KB of codes per
// 256-wide K step instead of 48 KB for the same tensor-core work (BN = 256),
// and the smaller stages fit five to a CTA instead of four.
//
// BN = 256 leaves room in TMEM for one accumulator: the MMAs of a tile wait
// until the epilogue has copied the previous tile's accumulator to registers.
//
// The pairs walk units: the first wide_tiles are whole tiles; when the tiles
// left over after the last full round are at most half as many as the pairs,
// each of them is split into two units of half its width (256 x 128, BN = 256
// only), so that twice as many pairs share that round, in half the time.  A
// half-width unit computes its columns exactly as the whole tile would: the
// same products, summed in the same order.
// BN = 192 fits two accumulators (TMEM columns 0 and 256) beside the scale
// factors, so the MMAs run on into the next tile while the epilogue drains the
// last one; it moves more operand bytes per MMA and pays where the K loop of a
// tile is short.
//
// Per CTA of the pair:
//   warp 0    : TMA producer for this CTA's stage buffers: A codes (128 x 128 B),
//               its half of B (BN / 2 x 128 B), the A scale atoms of its rows and
//               the B scale atoms of all BN columns (every CTA's TMEM needs
//               them), then the low-rank operands (its XL1 rows, its half of
//               [L2^T | L2^T]).  All of them count on rank 0's stage barrier;
//               rank 0 alone arms it with both CTAs' bytes.
//   warp 1    : TMEM (allocated for the pair); on rank 0 one lane moves both
//               CTAs' scales into their TMEM (tcgen05.cp.cta_group::2) and
//               issues the pair MMAs; each commit signals the matching barrier
//               in both CTAs.
//   warps 2-9 : epilogue of this CTA's 128 rows, as in gemm_nvfp4_kernel but
//               with 32-column TMA boxes (a 2 KB buffer per warp); the
//               hand-back of an accumulator counts on rank 0's barrier, which
//               waits for all sixteen epilogue warps of the pair.
#pragma once

#include "gemm_nvfp4.cuh"

namespace svdq {

constexpr int kPairBM = 256;                   // rows per pair tile (128 per CTA)
constexpr int kPairGroupM = 4;                 // pair row blocks per tile-order group
constexpr uint16_t kPairMask = 3;              // both CTAs of the pair

// Shape of the pair kernel for a tile width BN (weight columns per pair tile,
// BN / 2 per CTA).  BN = 256 keeps one accumulator in TMEM (256 columns of the
// 512, the scale factors in 48 more); BN = 192 fits two (columns 0 and 256),
// so the MMAs of the next tile need not wait for the epilogue to empty the
// last one.
template <int BN>
struct PairShape {
  static_assert(BN == 256 || BN == 192, "pair tiles are 256 or 192 columns wide");
  static constexpr int kBH = BN / 2;                                      // weight columns per CTA
  static constexpr int kAcc = BN == 256 ? 1 : 2;                          // accumulators in TMEM
  static constexpr int kStages = BN == 256 ? 5 : 6;
  static constexpr uint32_t kAOff = 0;                                    // 128 x 128 B
  static constexpr uint32_t kBOff = 128 * kGemmBKB;                       // kBH x 128 B
  static constexpr uint32_t kSfaOff = kBOff + kBH * kGemmBKB;             // 4 atoms
  static constexpr uint32_t kSfbOff = kSfaOff + 4 * 512;                  // 2 x 4 atoms
  static constexpr uint32_t kStageBytes = kSfbOff + 8 * 512;              // 38912 / 34816
  static constexpr uint32_t kEpiOff = kStageBytes * kStages;
  static constexpr uint32_t kEpiBufBytes = 32 * 64;                      // 32 rows x 32 bf16 per warp
  static constexpr uint32_t kBarOff = kEpiOff + kGemmEpiWarps * kEpiBufBytes;
  static constexpr uint32_t kSmemBytes = kBarOff + 256 + 1024;
  static constexpr uint32_t kAccStride = 256;                             // TMEM columns between accumulators
  static constexpr uint32_t kSfaCol = kAccStride * (kAcc - 1) + BN;       // 256 / 448
  static constexpr uint32_t kSfbCol = kSfaCol + 16;                       // 272 / 464
  static_assert(kStageBytes % 1024 == 0, "stage buffers keep the 1024-byte swizzle alignment");
  static_assert(kSfbCol + 32 <= kGemmTmemCols, "accumulators and scale factors fit in TMEM");
};
constexpr uint32_t kPairSmemBytes = PairShape<256>::kSmemBytes;
constexpr uint32_t kPair192SmemBytes = PairShape<192>::kSmemBytes;

// Epilogue store of the pair kernels: as epi_store_16 (gemm_nvfp4.cuh) for 32
// columns (n0 .. n0 + 31): a 2 KB buffer of 32 rows of 64 bytes
// in the TMA 64-byte swizzle (16-byte chunk c of row r at c ^ ((r >> 1) & 3)),
// one TMA store of the 32 x 32 box.  Used by the CTA-pair kernels: half the
// stores of 16-column boxes for the same bytes.
__device__ __forceinline__ void epi_store_32(const uint32_t* r, uint8_t* buf, const CUtensorMap* tm_y,
                                             int n0, int row0, int N,
                                             const __nv_bfloat16* __restrict__ bias, float out_scale,
                                             uint32_t lane) {
  uint32_t w[16];
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    float bb[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) bb[j] = 0.f;
    if (bias != nullptr && n0 + 8 * h < N) {
      const uint4 b = __ldg(reinterpret_cast<const uint4*>(bias + n0 + 8 * h));
      const uint32_t b4[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        bb[2 * t] = bf16_lo(b4[t]);
        bb[2 * t + 1] = bf16_hi(b4[t]);
      }
    }
#pragma unroll
    for (int t = 0; t < 4; ++t)
      w[4 * h + t] = pack_bf16x2(__fmaf_rn(__uint_as_float(r[8 * h + 2 * t]), out_scale, bb[2 * t]),
                                 __fmaf_rn(__uint_as_float(r[8 * h + 2 * t + 1]), out_scale, bb[2 * t + 1]));
  }
  if (lane == 0) bulk_wait_group_read<0>();   // the previous store has read the buffer
  __syncwarp();
  const uint32_t row_addr = smem_u32(buf) + lane * 64u;
  const uint32_t sw = (lane >> 1) & 3u;
#pragma unroll
  for (uint32_t c = 0; c < 4; ++c)
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row_addr + ((c ^ sw) << 4)),
                 "r"(w[4 * c]), "r"(w[4 * c + 1]), "r"(w[4 * c + 2]), "r"(w[4 * c + 3])
                 : "memory");
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tm_y, buf, n0, row0);
    bulk_commit_group();
  }
}

// Unit u of a pair's walk: units below p.wide_tiles are whole tiles in
// gemm_tile_coords order; tile p.wide_tiles + v / 2 of that order gives the
// units p.wide_tiles + v, the half v % 2 of its columns each.  Returns that
// half, or -1 for a whole tile.
__device__ __forceinline__ int pair_unit_coords(const GemmParams& p, int u, int& mp, int& nb) {
  if (u < p.wide_tiles) {
    gemm_tile_coords(p.m_tiles, p.n_tiles, p.group_m, u, mp, nb);
    return -1;
  }
  const int v = u - p.wide_tiles;
  gemm_tile_coords(p.m_tiles, p.n_tiles, p.group_m, p.wide_tiles + (v >> 1), mp, nb);
  return v & 1;
}

// p.m_tiles counts pair row blocks (256 rows), p.n_tiles weight column blocks
// of BN; p.sfa / p.sfb are unused (the scale atoms come through tm_sfa / tm_sfb:
// [atoms][128 x 32-bit words]; for tm_sfb, atom slot 2 nb + a of a K step holds
// the scales of weight columns nb BN + 128 a .. + 127).  tm_b and tm_l2t have
// boxes of BN / 2 rows; a half-width unit loads the same boxes from its own
// first column on and its MMAs read the first BN / 4 rows of each CTA's half.
template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_nvfp4_pair_kernel(const __grid_constant__ CUtensorMap tm_a,
                           const __grid_constant__ CUtensorMap tm_b,
                           const __grid_constant__ CUtensorMap tm_sfa,
                           const __grid_constant__ CUtensorMap tm_sfb,
                           const __grid_constant__ CUtensorMap tm_xl1,
                           const __grid_constant__ CUtensorMap tm_l2t,
                           const __grid_constant__ CUtensorMap tm_y, const GemmParams p) {
  using Sh = PairShape<BN>;
  constexpr int STAGES = Sh::kStages;
  constexpr int ACC = Sh::kAcc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Sh::kBarOff);   // rank 0's are used
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;                                 // [ACC]
  uint64_t* acc_empty = acc_full + ACC;                                // [ACC], rank 0's are used
  uint64_t* mma_done = acc_empty + ACC;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  // rank 0's copy: stages whose loads each CTA issued (read by rank 0's drain)
  uint32_t* issued = reinterpret_cast<uint32_t*>(tmem_holder + 2);

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
    for (int b = 0; b < ACC; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * kGemmEpiWarps);
    }
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
      const uint32_t main_tx = 2 * Sh::kStageBytes;
      const uint32_t lr_tx = 2 * (128 + Sh::kBH) * static_cast<uint32_t>(lr_cols) * 2;
      int it = 0;
      bool ok = true;
      for (int u = pair; u < p.num_units && ok; u += n_pairs) {
        int mp, nb;
        const int half = pair_unit_coords(p, u, mp, nb);
        const int m_blk = 2 * mp + static_cast<int>(rank);    // this CTA's 128-row block
        const int m0 = m_blk * 128;
        // this CTA's first weight column; the B scale atoms of the columns
        const int nh0 = half < 0 ? nb * BN + Sh::kBH * static_cast<int>(rank)
                                 : nb * BN + Sh::kBH * half + (Sh::kBH / 2) * static_cast<int>(rank);
        const int sfb0 = half < 0 ? 2 * nb : 2 * nb + half;
        const int sfb1 = half < 0 ? 2 * nb + 1 : 2 * nb + half;
        for (int step = 0; step < steps_per_tile; ++step, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, p.budget, abort_flag)) {
            raise_error(kErrWaitGemm);
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* st = smem + s * Sh::kStageBytes;
          const uint32_t fb = full0 + static_cast<uint32_t>(s) * 8u;
          if (step < p.kt_total) {
            const int kt = step;
            if (rank == 0) mbar_arrive_expect_tx(&full[s], main_tx);
            tma_load_2d_pair(st + Sh::kAOff, &tm_a, fb, kt * kGemmBKB, m0);
            tma_load_2d_pair(st + Sh::kBOff, &tm_b, fb, kt * kGemmBKB, nh0);
            tma_load_2d_pair(st + Sh::kSfaOff, &tm_sfa, fb, 0, m_blk * p.sf_kcols + 4 * kt);
            tma_load_2d_pair(st + Sh::kSfbOff, &tm_sfb, fb, 0, sfb0 * p.sf_kcols + 4 * kt);
            tma_load_2d_pair(st + Sh::kSfbOff + 2048, &tm_sfb, fb, 0, sfb1 * p.sf_kcols + 4 * kt);
          } else {
            const int c = step - p.kt_total;
            if (rank == 0) mbar_arrive_expect_tx(&full[s], lr_tx);
            tma_load_2d_pair(st + Sh::kAOff, &tm_xl1, fb, c * 64, m0);
            tma_load_2d_pair(st + Sh::kBOff, &tm_l2t, fb, c * 64, nh0);
          }
        }
      }
      // publish, in rank 0's shared memory, how many stages this CTA filled
      st_shared_cluster_u32(map_shared_rank(smem_u32(issued + rank), 0), static_cast<uint32_t>(it));
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (rank 0)
    if (rank == 0 && elect_one()) {
      const uint32_t idesc_main_w = idesc_e2m1_ue4m3(kPairBM, BN);
      const uint32_t idesc_lr_w = idesc_bf16_f32(kPairBM, BN);
      const uint32_t idesc_main_h = idesc_e2m1_ue4m3(kPairBM, BN / 2);   // half-width units
      const uint32_t idesc_lr_h = idesc_bf16_f32(kPairBM, BN / 2);
      const uint32_t lr_row_bytes = static_cast<uint32_t>(lr_cols) * 2;
      const uint32_t sfa_col = tmem_base + Sh::kSfaCol;
      const uint32_t sfb_col = tmem_base + Sh::kSfbCol;
      int it = 0, t_local = 0;
      bool ok = true;
      for (int u = pair; u < p.num_units && ok; u += n_pairs, ++t_local) {
        int mp, nb;
        const bool whole = pair_unit_coords(p, u, mp, nb) < 0;
        const uint32_t idesc_main = whole ? idesc_main_w : idesc_main_h;
        const uint32_t idesc_lr = whole ? idesc_lr_w : idesc_lr_h;
        // accumulator b of this unit; its previous unit's epilogue must have emptied it
        const int b = t_local % ACC;
        const uint32_t d_tmem = tmem_base + Sh::kAccStride * static_cast<uint32_t>(b);
        if (!mbar_wait(&acc_empty[b], ((t_local / ACC) & 1) ^ 1, p.budget, abort_flag)) {
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
          uint8_t* st = smem + s * Sh::kStageBytes;
          const uint32_t a0 = smem_u32(st + Sh::kAOff);
          const uint32_t b0 = smem_u32(st + Sh::kBOff);
          if (!tail) {
            const uint32_t sfa_s = smem_u32(st + Sh::kSfaOff);
            const uint32_t sfb_s = smem_u32(st + Sh::kSfbOff);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              tmem_cp_32x128b_x4_pair(sfa_col + 4 * j, sf_desc(sfa_s + 512 * j));
              tmem_cp_32x128b_x4_pair(sfb_col + 8 * j, sf_desc(sfb_s + 512 * j));
              tmem_cp_32x128b_x4_pair(sfb_col + 8 * j + 4, sf_desc(sfb_s + 2048 + 512 * j));
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              mma_nvf4_pair(d_tmem, make_kmajor_desc(a0 + 32 * j, 128), make_kmajor_desc(b0 + 32 * j, 128),
                            idesc_main, sfa_col + 4 * j, sfb_col + 8 * j, (step > 0 || j > 0) ? 1u : 0u);
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
        tc_commit_pair(&acc_full[b], kPairMask);
      }
      tc_commit_pair(mma_done, kPairMask);   // retires once every MMA and copy issued above has completed
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const uint32_t q = warp & 3u;
    const uint32_t h = (warp - 2) >> 2;
    constexpr int CH = Sh::kBH / 32;   // 32-column chunks of this warp's half of the tile
    uint8_t* ebuf = smem + Sh::kEpiOff + (warp - 2) * Sh::kEpiBufBytes;
    int t_local = 0;
    for (int u = pair; u < p.num_units; u += n_pairs, ++t_local) {
      int mp, nb;
      const int half = pair_unit_coords(p, u, mp, nb);
      // columns of this warp: half of the unit's BN (whole tile) or BN / 2 per CTA
      const int wcols = half < 0 ? Sh::kBH : Sh::kBH / 2;
      const int nch = wcols / 32;
      const int b = t_local % ACC;
      if (!warp_wait(&acc_full[b], (t_local / ACC) & 1, p.budget, abort_flag)) {
        if (lane == 0) raise_error(kErrWaitGemm);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      uint32_t v[CH][32];
      const uint32_t taddr = tmem_base + ((q * 32u) << 16) + Sh::kAccStride * static_cast<uint32_t>(b) +
                             static_cast<uint32_t>(wcols) * h;
#pragma unroll
      for (int c = 0; c < CH; ++c)
        if (c < nch) tmem_ld32(taddr + 32 * c, v[c]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_shared_rank(smem_u32(&acc_empty[b]), 0));
      const int row0 = mp * kPairBM + 128 * static_cast<int>(rank) + static_cast<int>(q) * 32;
      const int ncol = nb * BN + (half < 0 ? 0 : Sh::kBH * half) + wcols * static_cast<int>(h);
      if (row0 < p.M) {
#pragma unroll
        for (int c = 0; c < CH; ++c)
          if (c < nch && ncol + 32 * c < p.N)
            epi_store_32(v[c], ebuf, &tm_y, ncol + 32 * c, row0, p.N, p.bias, p.out_scale, lane);
      }
    }
    if (lane == 0) bulk_wait_group_all();
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();   // both producers have published their counts
  if (rank == 0 && threadIdx.x == 0) {
    // Drain: every load either CTA issued counts on rank 0's barriers and
    // writes into that CTA's shared memory, so none may still be in flight
    // when the pair leaves.  After a wait ran out the two producers may have
    // stopped at different stages: a stage only rank 1 filled is armed here
    // for rank 1's share, and in a stage only rank 0 filled rank 1's share is
    // completed without a copy.  Stages older than the last STAGES were all
    // consumed by the MMAs (a producer refills a buffer only after that).
    const int c0 = static_cast<int>(issued[0]), c1 = static_cast<int>(issued[1]);
    const int cmax = c0 > c1 ? c0 : c1;
    const uint32_t lr_share = (128 + Sh::kBH) * static_cast<uint32_t>(lr_cols) * 2;
    for (int i = (cmax > STAGES ? cmax - STAGES : 0); i < cmax; ++i) {
      uint64_t* bar = &full[i % STAGES];
      const uint32_t share = (i % steps_per_tile) < p.kt_total ? Sh::kStageBytes : lr_share;
      if (i >= c0)
        mbar_arrive_expect_tx(bar, share);
      else if (i >= c1)
        mbar_complete_tx(bar, share);
      if (!mbar_wait(bar, (i / STAGES) & 1, drain_budget(p.budget), nullptr)) raise_error(kErrWaitGemm);
    }
  }
  __syncthreads();
  if (warp == 1) {
    // every MMA of the pair has retired before its TMEM is released
    mbar_wait(mma_done, 0, drain_budget(p.budget), nullptr);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kGemmTmemCols);
  }
  // neither CTA leaves while the other may still signal its barriers or read
  // its shared memory
  cluster_sync();
}

}  // namespace svdq
