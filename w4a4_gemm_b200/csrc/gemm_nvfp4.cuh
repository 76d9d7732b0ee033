// gemm_nvfp4.cuh -- the fused 4-bit GEMM + low-rank up-projection + bias.
//
// SVDQuant Sec. 4.2 (Eq. 5) and Sec. 4.3 (Nunchaku, Fig. 6b):
//   Y = Q(X_hat) Q(R) + (X_hat L1) L2 + b
// The up-projection shares its output with the 4-bit GEMM, so its rank-r
// product is accumulated by the tensor core into the same TMEM accumulator
// right after the main K loop; the epilogue adds the bias and writes bf16 Y.
//
// Persistent kernel, one 128 x 256 output tile at a time per CTA:
//   warp 0    : TMA producer.  Per 256-wide K step: A codes (128 x 128 B),
//               B codes (256 x 128 B), the A / B scale atoms (bulk copies);
//               then the low-rank operands, XL1 (128 x 2r: the fp32 values as
//               bf16 hi | lo) and [L2^T | L2^T] (256 x 2r), so the tail MMA adds
//               (hi + lo) L2 with fp32 accuracy.
//   warp 1    : TMEM owner; one lane moves scales smem -> TMEM (tcgen05.cp)
//               and issues tcgen05.mma kind::mxf4nvf4 (E2M1 x E2M1, UE4M3
//               scale per 16) and, for the low-rank tail, kind::f16.
//   warps 2-9 : epilogue.  Warp w serves TMEM lane quarter w % 4 (rows) and
//               columns [128 h, 128 h + 128), h = (w - 2) / 4.  Per tile they
//               copy their accumulator columns to registers and hand the TMEM
//               back at once, so the next tile's MMAs overlap the bias, bf16
//               conversion and stores.  Each warp writes Y through its own 1 KB
//               shared-memory buffer (32 rows x 16 columns) and TMA stores:
//               whole 32-byte row segments instead of one scattered 16-byte
//               store per row and instruction, which kept the shared-memory
//               pipe busy while the tensor core was reading its operands.
#pragma once

#include "svdq_formats.cuh"
#include "svdq_ptx.cuh"

namespace svdq {

constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;
constexpr int kGemmBKB = 128;                  // K step in bytes of packed codes = 256 values
constexpr int kGemmThreads = 320;
constexpr int kGemmEpiWarps = 8;
constexpr uint32_t kGemmSfaCol = 256;          // 4 MMAs x 4 columns
constexpr uint32_t kGemmSfbCol = 272;          // 4 MMAs x 8 columns
constexpr uint32_t kGemmTmemCols = 512;

constexpr uint32_t kGemmAOff = 0;
constexpr uint32_t kGemmBOff = kGemmBM * kGemmBKB;                 // 16384
constexpr uint32_t kGemmSfaOff = kGemmBOff + kGemmBN * kGemmBKB;   // 49152
constexpr uint32_t kGemmSfbOff = kGemmSfaOff + 4 * 512;            // 51200
constexpr uint32_t kGemmStageBytes = kGemmSfbOff + 8 * 512;        // 55296

// Low-rank tail: its K (2 r_pad) is split into chunks of at most 64 bf16 (128 bytes).
__host__ __device__ inline int lr_chunk_cols(int k_tail) { return k_tail < 64 ? k_tail : 64; }
__host__ __device__ inline int lr_num_chunks(int k_tail) {
  return k_tail == 0 ? 0 : (k_tail + 63) / 64;
}
constexpr int kGemmStages = 4;
constexpr int kGemmGroupM = 8;                 // default tile-order group (gemm_tile_coords)
constexpr uint32_t kGemmEpiBufBytes = 32 * 32;                              // 32 rows x 16 bf16
constexpr uint32_t kGemmEpiOff = kGemmStageBytes * kGemmStages;
constexpr uint32_t kGemmBarOff = kGemmEpiOff + kGemmEpiWarps * kGemmEpiBufBytes;
constexpr uint32_t kGemmSmemBytes = kGemmBarOff + 256 + 1024;

struct GemmParams {
  int M, N, K;
  int kt_total;        // ceil(K / 256)
  int m_tiles, n_tiles, num_tiles;
  int group_m;         // tile order: groups of group_m row blocks, see gemm_tile_coords
  int wide_tiles;      // CTA-pair kernels: tiles taken whole; each later one as two half-width units
  int num_units;       // CTA-pair kernels: wide_tiles + 2 (num_tiles - wide_tiles)
  int r_tail;          // tail K: 2 r_pad (X_hat L1 as hi | lo against L2^T | L2^T), 0 = none
  const uint8_t* sfa;  // activation scale atoms [M_pad/128][sf_kcols][512]
  const uint8_t* sfb;  // weight scale atoms     [N_pad/128][sf_kcols][512]
  int sf_kcols;        // K_pad / 64, K_pad = K rounded up to 256
  const __nv_bfloat16* bias;  // N or nullptr
  float out_scale;     // 2^-e of the weight prescale: y = acc * out_scale + b (exact scaling)
  long long budget;
};

// Tile order of the persistent kernels: the row blocks form groups of group_m
// (the last group may be shorter); a group's tiles come before the next
// group's, and within a group consecutive tiles walk down its row blocks for a
// fixed column block of the weights.  The tiles in flight at one time (one per
// CTA) then read about gridDim / group_m weight column blocks and group_m
// activation row blocks, which keeps the operands they share resident in L2.
// group_m = m_tiles walks all of M for each weight column block.  The default,
// kGemmGroupM row blocks, keeps both operands' working sets small at every
// layer shape of the FLUX block: the long-K MLP down-projection (K = 12288,
// 16384 rows) walking all of M re-reads its 100 MB of activation codes from
// DRAM for every weight column block and runs 22 % slower.
__device__ __forceinline__ void gemm_tile_coords(int m_tiles, int n_tiles, int group_m, int tile,
                                                 int& m_blk, int& n_blk) {
  const int span = group_m * n_tiles;
  const int g = tile / span;
  const int r = tile - g * span;
  const int first = g * group_m;
  const int rows = min(group_m, m_tiles - first);
  m_blk = first + r % rows;
  n_blk = r / rows;
}

__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
  // 32 rows x 16 bytes, rows 16 bytes apart, 8-row groups 128 bytes apart
  return make_sdesc(saddr, 0, 128, kSwizzleNone);
}

// Epilogue: 16 fp32 accumulators of this lane's row (columns n0 .. n0 + 15)
// times out_scale (a power of two: exact) + bias -> bf16 -> the warp's buffer (32 rows of 32 bytes in the TMA 32-byte
// swizzle: the 16-byte half c of row r sits at half c ^ ((r >> 2) & 1)) ->
// one TMA store of the 32 x 16 box at (n0, row0).  The store clips rows past M
// and columns past N; the bias is read only below N (N % 16 == 0).
__device__ __forceinline__ void epi_store_16(const uint32_t* r, uint8_t* buf, const CUtensorMap* tm_y,
                                             int n0, int row0, int N,
                                             const __nv_bfloat16* __restrict__ bias, float out_scale,
                                             uint32_t lane) {
  float bb[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) bb[j] = 0.f;
  if (bias != nullptr && n0 < N) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 b = __ldg(reinterpret_cast<const uint4*>(bias + n0 + 8 * h));
      const uint32_t b4[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        bb[8 * h + 2 * t] = bf16_lo(b4[t]);
        bb[8 * h + 2 * t + 1] = bf16_hi(b4[t]);
      }
    }
  }
  uint32_t w[8];
#pragma unroll
  for (int t = 0; t < 8; ++t)
    w[t] = pack_bf16x2(__fmaf_rn(__uint_as_float(r[2 * t]), out_scale, bb[2 * t]),
                       __fmaf_rn(__uint_as_float(r[2 * t + 1]), out_scale, bb[2 * t + 1]));
  if (lane == 0) bulk_wait_group_read<0>();   // the previous store has read the buffer
  __syncwarp();
  const uint32_t row_addr = smem_u32(buf) + lane * 32u;
  const uint32_t sw = (lane >> 2) & 1u;
#pragma unroll
  for (uint32_t c = 0; c < 2; ++c)
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

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tm_a,
                      const __grid_constant__ CUtensorMap tm_b,
                      const __grid_constant__ CUtensorMap tm_xl1,
                      const __grid_constant__ CUtensorMap tm_l2t,
                      const __grid_constant__ CUtensorMap tm_y, const GemmParams p) {
  constexpr int STAGES = kGemmStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGemmBarOff);
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
    mbar_init(acc_empty, kGemmEpiWarps);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kGemmTmemCols);
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
      const uint32_t lr_tx = (kGemmBM + kGemmBN) * lr_cols * 2;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        int m_blk, n_blk;
        gemm_tile_coords(p.m_tiles, p.n_tiles, p.group_m, tile, m_blk, n_blk);
        const int m0 = m_blk * kGemmBM, n0 = n_blk * kGemmBN;
        for (int step = 0; step < steps_per_tile; ++step, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, p.budget, abort_flag)) {
            raise_error(kErrWaitGemm);
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kGemmStageBytes;
          if (step < p.kt_total) {
            const int kt = step;
            mbar_arrive_expect_tx(&full[s], kGemmStageBytes);
            tma_load_2d(st + kGemmAOff, &tm_a, &full[s], kt * kGemmBKB, m0);
            tma_load_2d(st + kGemmBOff, &tm_b, &full[s], kt * kGemmBKB, n0);
            bulk_load(st + kGemmSfaOff,
                      p.sfa + (static_cast<size_t>(m_blk) * p.sf_kcols + kt * 4) * 512, 2048,
                      &full[s]);
            bulk_load(st + kGemmSfbOff,
                      p.sfb + (static_cast<size_t>(2 * n_blk) * p.sf_kcols + kt * 4) * 512, 2048,
                      &full[s]);
            bulk_load(st + kGemmSfbOff + 2048,
                      p.sfb + (static_cast<size_t>(2 * n_blk + 1) * p.sf_kcols + kt * 4) * 512,
                      2048, &full[s]);
          } else {
            const int c = step - p.kt_total;
            mbar_arrive_expect_tx(&full[s], lr_tx);
            tma_load_2d(st + kGemmAOff, &tm_xl1, &full[s], c * 64, m0);
            tma_load_2d(st + kGemmBOff, &tm_l2t, &full[s], c * 64, n0);
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
      const uint32_t idesc_main = idesc_e2m1_ue4m3(kGemmBM, kGemmBN);
      const uint32_t idesc_lr = idesc_bf16_f32(kGemmBM, kGemmBN);
      const uint32_t lr_row_bytes = static_cast<uint32_t>(lr_cols) * 2;
      const uint32_t d_tmem = tmem_base;
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
          const bool tail = step >= p.kt_total;
          if (!mbar_wait(&full[s], ph, p.budget, abort_flag)) {
            raise_error(kErrWaitGemm);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* st = smem + s * kGemmStageBytes;
          const uint32_t a0 = smem_u32(st + kGemmAOff);
          const uint32_t b0 = smem_u32(st + kGemmBOff);
          if (!tail) {
            const uint32_t sfa_s = smem_u32(st + kGemmSfaOff);
            const uint32_t sfb_s = smem_u32(st + kGemmSfbOff);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              tmem_cp_32x128b_x4(tmem_base + kGemmSfaCol + 4 * j, sf_desc(sfa_s + 512 * j));
              tmem_cp_32x128b_x4(tmem_base + kGemmSfbCol + 8 * j, sf_desc(sfb_s + 512 * j));
              tmem_cp_32x128b_x4(tmem_base + kGemmSfbCol + 8 * j + 4,
                                 sf_desc(sfb_s + 2048 + 512 * j));
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              mma_nvf4(d_tmem, make_kmajor_desc(a0 + 32 * j, 128), make_kmajor_desc(b0 + 32 * j, 128),
                       idesc_main, tmem_base + kGemmSfaCol + 4 * j, tmem_base + kGemmSfbCol + 8 * j,
                       (step > 0 || j > 0) ? 1u : 0u);
            }
          } else {
            for (int j = 0; j < lr_cols / 16; ++j) {
              mma_bf16(d_tmem, make_kmajor_desc(a0 + 32 * j, lr_row_bytes),
                       make_kmajor_desc(b0 + 32 * j, lr_row_bytes), idesc_lr, 1u);
            }
          }
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
      tc_commit(mma_done);  // retires once every MMA and copy issued above has completed
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const uint32_t q = warp & 3u;
    const uint32_t h = (warp - 2) >> 2;
    uint8_t* ebuf = smem + kGemmEpiOff + (warp - 2) * kGemmEpiBufBytes;
    int t_local = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++t_local) {
      int m_blk, n_blk;
      gemm_tile_coords(p.m_tiles, p.n_tiles, p.group_m, tile, m_blk, n_blk);
      // accumulator columns [128 h, 128 h + 128) of this warp's 32 rows -> registers
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
      if (lane == 0) mbar_arrive(acc_empty);
      // bias, bf16, staged TMA stores
      const int row0 = m_blk * kGemmBM + static_cast<int>(q) * 32;
      const int nb = n_blk * kGemmBN + 128 * static_cast<int>(h);
      if (row0 < p.M) {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (nb + 16 * c < p.N)
            epi_store_16(&v[c / 2][16 * (c % 2)], ebuf, &tm_y, nb + 16 * c, row0, p.N, p.bias, p.out_scale,
                         lane);
      }
    }
    if (lane == 0) bulk_wait_group_all();
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // every MMA issued by this CTA has retired before its TMEM is released
    mbar_wait(mma_done, 0, drain_budget(p.budget), nullptr);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kGemmTmemCols);
  }
}

}  // namespace svdq
