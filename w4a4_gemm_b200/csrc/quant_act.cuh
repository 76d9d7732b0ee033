// quant_act.cuh -- the fused activation kernel: smoothing, per-group 4-bit
// quantization and the low-rank down-projection in one pass over X.
//
// SVDQuant Sec. 4.3 (Nunchaku, Fig. 6b): the down-projection X_hat L1 shares
// its input with the quantizer, so both are computed from one read of X.  The
// smoothing is folded into the factor, X_hat L1 = X (diag(lambda)^-1 L1), so
// the tensor core reads the TMA-loaded X tile as it is, in parallel with the
// quantizer warps.  One bf16 rounding of the folded factor (2^-8 per term)
// would move Y by several times the output tolerance where the branch and the
// 4-bit part cancel, so the factor is carried as a bf16 pair L1s = hi + lo
// (2^-16 per term): the lo slices sit right after the hi slices in the stage,
// and one MMA of twice the width (two where that exceeds N = 256) puts X hi and
// X lo side by side in the accumulator, summed in fp32 at the end (bf16 x bf16
// products are exact in fp32).
//
// A cluster of C CTAs owns BM = 128 / S token rows; its CTA of rank t takes
// the t-th of C consecutive K ranges.  Each pipeline stage holds S consecutive
// 64-wide K sub-tiles of those rows stacked on top of each other as the
// 128-row A operand of one tcgen05 MMA, and the S matching 64 x r_pad slices
// of the folded factor L1s side by side as its N = S * r_pad wide B operand
// (once for hi, then once for lo, at column offset S * r_pad):
//   D[j*BM + i, j'*r_pad + c] += sum_k x[i, sub-tile j, k] * L1s[sub-tile j', k, c]
// Only the diagonal blocks j == j' are wanted; summing them over j and over
// the cluster's K ranges gives X L1s = X_hat L1 for row i.  The partial sums
// meet in distributed shared memory: each CTA parks its blocks in its own
// shared memory and sums, for its share of the rows, every CTA's blocks in a
// fixed order (the result does not depend on timing).  Codes and scales are
// local to a 64-wide group and need no exchange.
//
// Every stage carries L1s as well as X: 2 r_pad / BM bytes of factor (hi and
// lo) per byte of X.  Stacking (S > 1) fills the MMA at small M but raises
// that ratio; the K split (C > 1) keeps BM large and still gives every SM a
// CTA.  The host picks (S, C) from the SM count and the resident clusters of
// each size.
//   warp 0      : TMA producer (S X boxes BM x 64, 2 S L1s^T boxes r_pad x 64
//                 (hi, lo), 1/lambda)
//   warp 1      : TMEM owner; one lane issues the kind::f16 MMAs
//   warps 2..17 : quantizers in up to four groups of four (as many groups as
//                 there are pipeline stages); group k takes every G-th stage,
//                 and its warp w serves A-tile rows 32 (w % 4) .. + 31, one lane
//                 per row over the whole 64-wide sub-tile.  They smooth X,
//                 quantize it, release the stage and store codes and scales.
//                 At the end warps 2..5 read the diagonal blocks and the CTA
//                 sums them into XL1, kept at fp32 precision as a bf16 pair
//                 hi + lo for the GEMM's tail MMA.
#pragma once

#include "svdq_formats.cuh"
#include "svdq_ptx.cuh"

namespace svdq {

constexpr int kQuantTileRows = 128;   // rows of the MMA A operand
constexpr int kQuantBK = 64;          // K width of one sub-tile
constexpr int kQuantMaxStages = 12;
constexpr int kQuantMaxSplit = 8;     // CTAs per cluster splitting K
constexpr int kQuantGroups = 4;       // quantizer groups working on consecutive stages (at most)
constexpr int kQuantGroupWarps = 4;   // warps per group: one lane per row of a 128-row stage
constexpr int kQuantWarps = kQuantGroupWarps * kQuantGroups;
constexpr int kQuantThreads = 32 * (2 + kQuantWarps);
constexpr uint32_t kQuantSmemBudget = 220u * 1024u;    // shared memory for stages + code staging

// Bytes of codes one row of a 64-wide sub-tile produces: 64 E2M1 (NVFP4, FP4 g32) or 64 int8 (INT4, W8A8).
__host__ __device__ constexpr uint32_t quant_code_row_bytes(int fmt) { return (fmt == 1 || fmt == 3) ? 64u : 32u; }

struct QuantParams {
  int M, K;
  int r_pad;        // 0 = no low-rank branch; else 16, 32, 64, 128, 192 or 256
  int S;            // stacked K sub-tiles per stage (BM = 128 / S rows per cluster)
  int C;            // CTAs per cluster, each on its own K range (1, 2, 4 or 8; C <= BM)
  int per;          // stages per cluster rank: rank t takes stages [t per, min((t+1) per, total))
  int M_pad;        // M rounded up to 128 (scale atoms)
  int sf_kcols;     // NVFP4: K_pad / 64 scale atoms per 128-row block
  const float* inv_lambda;  // K rounded up to 512 (zero padded)
  uint8_t* sf;      // NVFP4: 512-byte atoms; INT4: fp16 [K/64][M_pad]
  __nv_bfloat16* xl1;  // M x 2 r_pad: X_hat L1 as a bf16 pair, hi | lo (hi + lo = fp32 value)
  long long budget;
};

// Most sub-tiles that can be stacked for a given padded rank (N = S * r_pad <= 256).
__host__ __device__ inline int quant_stack_max(int r_pad) {
  if (r_pad <= 32) return 8;
  if (r_pad <= 64) return 4;
  if (r_pad <= 128) return 2;
  return 1;
}

struct QuantSmem {
  uint32_t x_off, l1_off, il_off, stage_bytes, stages, groups, stg_off, stg_bytes, bar_off, total;
};

// Per stage: the stacked X tile, S slices of L1s^T hi then S of lo, and
// 1/lambda.  After the stages: one code staging buffer (32 rows of codes) per
// quantizer warp.
// G groups take the stages in turn, and the buffer count is a multiple of G,
// so stage buffer b always serves group b mod G; G is 4 or 3, whichever keeps
// more of the buffers that fit (4 on a tie: the quantizers set the pace), or
// the buffer count itself when fewer than three fit.  A group
// waits on its next stage by the one-bit phase parity of the buffer's full
// barrier; that parity is unambiguous only if the buffer's previous fill has
// landed, which holds when that previous fill was this group's own stage.
// (With buffers shared between groups, a group could wait while another
// group's stage was still in flight to the same buffer -- TMA fills complete
// out of order under load -- and match the phase before it.)
__host__ __device__ inline QuantSmem quant_smem_layout(int fmt, int r_pad, int S) {
  QuantSmem L;
  L.x_off = 0;
  L.l1_off = kQuantTileRows * kQuantBK * 2;                // 16384
  L.il_off = L.l1_off + 2 * S * r_pad * 128;               // 2 S r_pad rows of 128 bytes (hi, lo)
  uint32_t sb = L.il_off + S * kQuantBK * 4;
  L.stage_bytes = (sb + 1023u) & ~1023u;
  L.stg_bytes = 32u * quant_code_row_bytes(fmt);           // one staging buffer: a warp's 32 rows
  const uint32_t stg_total = kQuantWarps * L.stg_bytes;
  L.stages = (kQuantSmemBudget - stg_total) / L.stage_bytes;
  if (L.stages > static_cast<uint32_t>(kQuantMaxStages)) L.stages = kQuantMaxStages;
  if (L.stages < 3u) {
    L.groups = L.stages;
  } else {
    static_assert(kQuantGroups == 4, "the group rule below picks 4 or 3 groups");
    L.groups = (L.stages - L.stages % 4u) >= (L.stages - L.stages % 3u) ? 4u : 3u;
  }
  if (L.groups > 0) L.stages -= L.stages % L.groups;
  L.stg_off = L.stage_bytes * L.stages;
  L.bar_off = L.stg_off + stg_total;
  L.total = L.bar_off + 256 + 512 + 1024;                  // barriers, 1/scale table, alignment
  return L;
}

template <int FMT>  // 0 = NVFP4 (groups of 16), 1 = INT4 (groups of 64), 2 = FP4 g32 (groups of 32),
                    // 3 = W8A8 (int8, the per-token scale computed beforehand by w8_row_scale_kernel)
__global__ void __launch_bounds__(kQuantThreads, 1)
    quant_act_kernel(const __grid_constant__ CUtensorMap tm_x,
                     const __grid_constant__ CUtensorMap tm_l1t,
                     const __grid_constant__ CUtensorMap tm_codes, const QuantParams p) {
  extern __shared__ uint8_t smem_raw[];
  const QuantSmem L = quant_smem_layout(FMT, p.r_pad, p.S);
  uint8_t* smem = align_smem_1024(smem_raw);
  const int NS = static_cast<int>(L.stages);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* empty = full + kQuantMaxStages;
  uint64_t* acc_full = empty + kQuantMaxStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* rcp_tab = reinterpret_cast<float*>(smem + L.bar_off + 256);   // 1/E4M3 value, 128 entries

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const bool has_lr = p.r_pad > 0;
  const int S = p.S;
  const int BM = kQuantTileRows / S;
  const int rank = static_cast<int>(blockIdx.x) % p.C;  // rank in the 1-D cluster of C CTAs
  const int m0 = (static_cast<int>(blockIdx.x) / p.C) * BM;
  const int kstep = S * kQuantBK;                       // K columns per stage
  const int nkt = (p.K + kstep - 1) / kstep;            // stages over all of K
  const int i0 = min(rank * p.per, nkt);                // this CTA's stages: i0 .. i0 + n_local - 1
  const int n_local = min(nkt - i0, p.per);
  const int n_mma = S * p.r_pad;                        // columns of the hi (and of the lo) product
  // the accumulator: hi products in columns 0 .. n_mma - 1, lo in n_mma .. 2 n_mma - 1
  const uint32_t tmem_cols = n_mma <= 16 ? 32u : (n_mma <= 32 ? 64u : (n_mma <= 64 ? 128u : (n_mma <= 128 ? 256u : 512u)));

  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      // released by the quantizer warps and, with a low-rank branch, the MMAs
      mbar_init(&empty[s], kQuantGroupWarps + (has_lr ? 1 : 0));
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if ((FMT == 0 || FMT == 2) && warp >= 2 && warp < 6) fill_e4m3_rcp_table(rcp_tab, threadIdx.x - 64, 128);
  if (warp == 1 && has_lr) {
    tmem_alloc(tmem_holder, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = has_lr ? *tmem_holder : 0u;
  // X and the previous contents of the workspace belong to earlier kernels
  griddep_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      prefetch_tmap(&tm_x);
      if (has_lr) prefetch_tmap(&tm_l1t);
      const uint32_t tx = S * (BM * kQuantBK * 2 + (has_lr ? 2 * p.r_pad * 128 : 0) + kQuantBK * 4);
      int issued = 0;
      for (int li = 0; li < n_local; ++li) {
        const int i = i0 + li;
        const int s = li % NS;
        const uint32_t ph = (li / NS) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, p.budget, abort_flag)) {
          raise_error(kErrWaitQuant);
          *abort_flag = 1;
          break;
        }
        uint8_t* st = smem + s * L.stage_bytes;
        mbar_arrive_expect_tx(&full[s], tx);
        for (int j = 0; j < S; ++j) {
          const int k = (i * S + j) * kQuantBK;   // may lie past K: the box is zero-filled
          tma_load_2d(st + L.x_off + j * BM * 128, &tm_x, &full[s], k, m0);
          if (has_lr) {   // rows 0 .. r_pad - 1 of the map hold hi, r_pad .. 2 r_pad - 1 lo
            tma_load_2d(st + L.l1_off + j * p.r_pad * 128, &tm_l1t, &full[s], k, 0);
            tma_load_2d(st + L.l1_off + (S + j) * p.r_pad * 128, &tm_l1t, &full[s], k, p.r_pad);
          }
        }
        bulk_load(st + L.il_off, p.inv_lambda + i * kstep, S * kQuantBK * 4, &full[s]);
        issued = li + 1;
      }
      // never leave while a copy into this CTA's shared memory is still in flight
      // (whether or not a wait ran out, and in whichever role)
      for (int i = (issued > NS ? issued - NS : 0); i < issued; ++i)
        mbar_wait(&full[i % NS], (i / NS) & 1, drain_budget(p.budget), nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (has_lr && elect_one()) {
      // one MMA of N = 2 n_mma over the hi and lo slices (adjacent in the
      // stage) where N fits, else one for each
      const bool one = 2 * n_mma <= 256;
      const uint32_t idesc = idesc_bf16_f32(kQuantTileRows, one ? 2 * n_mma : n_mma);
      for (int li = 0; li < n_local; ++li) {
        const int s = li % NS;
        const uint32_t ph = (li / NS) & 1;
        if (!mbar_wait(&full[s], ph, p.budget, abort_flag)) {
          raise_error(kErrWaitQuant);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + s * L.stage_bytes + L.x_off);
        const uint32_t b0 = smem_u32(smem + s * L.stage_bytes + L.l1_off);   // hi slices
        const uint32_t b1 = b0 + static_cast<uint32_t>(S * p.r_pad * 128);    // lo slices
#pragma unroll
        for (int k = 0; k < kQuantBK / 16; ++k) {
          mma_bf16(tmem_base, make_kmajor_desc(a0 + 32 * k, 128), make_kmajor_desc(b0 + 32 * k, 128),
                   idesc, (li > 0 || k > 0) ? 1u : 0u);
        }
        if (!one) {
#pragma unroll
          for (int k = 0; k < kQuantBK / 16; ++k)
            mma_bf16(tmem_base + static_cast<uint32_t>(n_mma), make_kmajor_desc(a0 + 32 * k, 128),
                     make_kmajor_desc(b1 + 32 * k, 128), idesc, (li > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(&empty[s]);
      }
      tc_commit(acc_full);  // also covers an early exit: waits for every issued MMA
    }
  } else {
    // ------------------------------------------------------------ quantizers
    // Group k = (warp - 2) / 4 takes the stages k, k + G, k + 2G, ... (G active
    // groups; stage buffer b always serves group b mod G, see quant_smem_layout);
    // its warp of lane quarter q quantizes rows 32 q .. 32 q + 31 of the
    // stacked tile, one lane per row over the whole 64-wide sub-tile: four
    // independent NVFP4 groups of 16 (or one INT4 group of 64) per lane.  Each
    // warp stages its own 32 rows of codes in shared memory (one buffer, which
    // its previous store has read long before the next stage) and its lane 0
    // writes them with one TMA store per sub-tile the
    // rows belong to (boxes of min(32, BM) rows), so no barrier ties the warps
    // of a group together; each lane writes its row's scales itself (one 4-byte
    // word or one fp16).
    constexpr uint32_t RB = quant_code_row_bytes(FMT);   // code bytes per row
    const uint32_t q = warp & 3u;
    const int grp = static_cast<int>(warp - 2) >> 2;
    const uint32_t R = q * 32 + lane;          // row of the stacked A tile
    const int st_boxes = BM < 32 ? 2 : 1;                               // code stores per stage
    const int st_j0 = static_cast<int>(q * 32) / BM;                    // sub-tile of the first box
    const int st_m0 = m0 + static_cast<int>(q * 32) % BM;               // its first token row
    const int j = static_cast<int>(R) / BM;    // K sub-tile
    const int m = m0 + static_cast<int>(R) % BM;
    const bool row_ok = m < p.M;
    float w8_inv = 0.0f;   // W8A8: 1 / this row's token scale, fixed for every stage
    if constexpr (FMT == 3) {
      const float sd = reinterpret_cast<const float*>(p.sf)[row_ok ? m : 0];
      w8_inv = (sd == 0.0f || !row_ok) ? 0.0f : __frcp_rn(sd);
    }
    const int G = static_cast<int>(L.groups);
    for (int li = grp < G ? grp : n_local; li < n_local; li += G) {
      const int i = i0 + li;
      const int s = li % NS;
      const uint32_t ph = (li / NS) & 1;
      const bool ok = warp_wait(&full[s], ph, p.budget, abort_flag);
      if (!ok) {
        if (lane == 0) raise_error(kErrWaitQuant);
        *abort_flag = 1;
      }
      const int kcol = i * S + j;              // 64-wide column group of X
      const bool col_ok = kcol * kQuantBK < p.K;
      const uint8_t* st = smem + s * L.stage_bytes;
      float v[64];
      if (ok) {
        const float4* il = reinterpret_cast<const float4*>(st + L.il_off + j * kQuantBK * 4);
        const uint8_t* xrow = st + L.x_off + R * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t chunk = (static_cast<uint32_t>(c) ^ (R & 7u)) << 4;   // 128-byte swizzle
          const uint4 raw = *reinterpret_cast<const uint4*>(xrow + chunk);
          const float4 l0 = il[2 * c], l1 = il[2 * c + 1];
          float2 t;
          t = fmul2_rn(make_float2(bf16_lo(raw.x), bf16_hi(raw.x)), make_float2(l0.x, l0.y));
          v[8 * c + 0] = t.x; v[8 * c + 1] = t.y;
          t = fmul2_rn(make_float2(bf16_lo(raw.y), bf16_hi(raw.y)), make_float2(l0.z, l0.w));
          v[8 * c + 2] = t.x; v[8 * c + 3] = t.y;
          t = fmul2_rn(make_float2(bf16_lo(raw.z), bf16_hi(raw.z)), make_float2(l1.x, l1.y));
          v[8 * c + 4] = t.x; v[8 * c + 5] = t.y;
          t = fmul2_rn(make_float2(bf16_lo(raw.w), bf16_hi(raw.w)), make_float2(l1.z, l1.w));
          v[8 * c + 6] = t.x; v[8 * c + 7] = t.y;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 64; ++e) v[e] = 0.0f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);   // X of this stage is in registers
      uint32_t out[RB / 4];
      uint32_t sfw;
      if constexpr (FMT == 0) {
        sfw = 0;
#pragma unroll
        for (int g = 0; g < 4; ++g) sfw |= quant16_nvfp4(v + 16 * g, out + 2 * g, rcp_tab) << (8 * g);
      } else if constexpr (FMT == 2) {
        // one scale per 32 values, stored in both 16-value slots of the atom
        const uint32_t s0 = quant32_fp4(v, out, rcp_tab);
        const uint32_t s1 = quant32_fp4(v + 32, out + 4, rcp_tab);
        sfw = s0 * 0x0101u | (s1 * 0x0101u) << 16;
      } else if constexpr (FMT == 3) {
        // int8 codes of this row with its per-token scale
        const float inv = w8_inv;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          uint32_t w = 0;
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int q = max(-127, min(127, __float2int_rn(__fmul_rn(v[4 * e + b], inv))));
            w |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * b);
          }
          out[e] = w;
        }
        sfw = 0;
      } else {
        float amax = 0.0f;
#pragma unroll
        for (int e = 0; e < 64; e += 16) amax = fmaxf(amax, absmax16(v + e));
        const uint16_t sh = int4_scale_bits(amax);
        const float sd = __half2float(__ushort_as_half(sh));
        const float inv = sd == 0.0f ? 0.0f : __frcp_rn(sd);
        // int8 codes in the INT4 GEMM's K order: in each run of eight values the
        // even positions first, then the odd ones (the order in which the GEMM
        // unpacks the 4-bit weight codes)
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int base = 8 * (e >> 1) + (e & 1);
          uint32_t w = 0;
#pragma unroll
          for (int b = 0; b < 4; ++b)
            w |= (static_cast<uint32_t>(int4_code(v[base + 2 * b], inv)) & 0xFFu) << (8 * b);
          out[e] = sd == 0.0f ? 0u : w;
        }
        sfw = sh;
      }
      // codes -> this warp's staging buffer (rows of RB bytes in the TMA swizzle
      // of that row length: 16-byte chunk c of row r sits at c ^ ((r >> sh) & mask))
      uint8_t* buf = smem + L.stg_off + (warp - 2) * L.stg_bytes;
      if (lane == 0) bulk_wait_group_read<0>();   // its store of the previous stage has read it
      __syncwarp();
      {
        const uint32_t row_addr = smem_u32(buf) + lane * RB;
        const uint32_t sw = RB == 32 ? ((lane >> 2) & 1u) : ((lane >> 1) & 3u);
#pragma unroll
        for (uint32_t c = 0; c < RB / 16; ++c)
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row_addr + ((c ^ sw) << 4)),
                       "r"(out[4 * c]), "r"(out[4 * c + 1]), "r"(out[4 * c + 2]), "r"(out[4 * c + 3])
                       : "memory");
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && ok) {
        // rows 32 q .. 32 q + 31 of the stacked tile: one box of 32 rows, or
        // (BM = 16) two boxes in consecutive sub-tiles
        for (int b = 0; b < st_boxes; ++b) {
          const int kc = i * S + st_j0 + b;
          if (kc * kQuantBK < p.K) tma_store_2d(&tm_codes, buf + b * 16 * RB, kc * RB, st_m0);
        }
        bulk_commit_group();
      }
      if (ok && col_ok && FMT != 3) {   // W8A8 scales are written before this kernel
        if constexpr (FMT == 0 || FMT == 2) {
          // scale atom: 128 rows x 4 scales, byte (m % 32) * 16 + (m % 128 / 32) * 4 + k4
          uint8_t* atom = p.sf + (static_cast<size_t>(m / 128) * p.sf_kcols + kcol) * 512;
          *reinterpret_cast<uint32_t*>(atom + (m & 31) * 16 + ((m & 127) >> 5) * 4) = row_ok ? sfw : 0u;
        } else {
          reinterpret_cast<uint16_t*>(p.sf)[static_cast<size_t>(kcol) * p.M_pad + m] =
              row_ok ? static_cast<uint16_t>(sfw) : static_cast<uint16_t>(0);
        }
      }
    }
    if (lane == 0) bulk_wait_group_all();
  }
  __syncwarp();

  // ---------------------------------------------------------------- XL1 out
  // Diagonal block j of the accumulator = the K sub-tiles j (mod S) of this
  // CTA's K range; warps 2..5 park them in shared memory over the first stage
  // buffers.  Those are free only once every quantizer group has read its last
  // stage (the accumulator is complete as soon as the last stage has landed,
  // and another group may still be reading a late stage in buffer 0): hence
  // the CTA barrier first.  Then each CTA of the cluster takes BM / C of the
  // rows and sums, for them, the parked blocks of every CTA (rank 0 first)
  // over j in fixed order, and rounds to bf16.
  // [128][r_pad + 4] fp32: the 16-byte pad puts consecutive rows on different
  // banks, so the lanes' row-wise float4 stores do not conflict
  float* red = reinterpret_cast<float*>(smem);
  const int rs = p.r_pad + 4;
  __syncthreads();
  if (has_lr && warp >= 2 && warp < 6) {
    const uint32_t q = warp & 3u;
    const uint32_t R = q * 32 + lane;
    const int j = static_cast<int>(R) / BM;
    if (!warp_wait(acc_full, 0, p.budget, abort_flag)) {
      if (lane == 0) raise_error(kErrWaitQuant);
      *abort_flag = 1;
    }
    tc_fence_after();
    // a TMEM load reads the same columns for all 32 lanes: when a warp's rows
    // span two sub-tiles (BM = 16), read both diagonal blocks, keep the own one
    const int j_first = static_cast<int>(q * 32) / BM, j_last = static_cast<int>(q * 32 + 31) / BM;
    for (int jj = j_first; jj <= j_last; ++jj) {
      for (int c = 0; c < p.r_pad; c += 16) {
        // the hi and the lo product of the block, summed in fp32
        uint32_t r[16], rl[16];
        if (n_local > 0) {
          tmem_ld16(tmem_base + ((q * 32u) << 16) + jj * p.r_pad + c, r);
          tmem_ld16(tmem_base + ((q * 32u) << 16) + n_mma + jj * p.r_pad + c, rl);
          tmem_wait_ld();
        } else {   // an empty K range contributes zero (its accumulator was never written)
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = rl[e] = 0u;
        }
        if (jj == j) {
          float v[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = __fadd_rn(__uint_as_float(r[e]), __uint_as_float(rl[e]));
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<float4*>(red + R * rs + c + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
      }
    }
  }
  tc_fence_before();
  cluster_sync();   // every CTA of the cluster has parked its blocks (C = 1: the CTA)
  if (has_lr) {
    // this CTA's BM / C rows x r_pad columns, 8 columns per thread over all threads
    const int rows = BM / p.C;
    const int units = rows * (p.r_pad / 8);
    for (int u = threadIdx.x; u < units; u += kQuantThreads) {
      const int i = rank * rows + u / (p.r_pad / 8);
      const int c = (u % (p.r_pad / 8)) * 8;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int t = 0; t < p.C; ++t) {
        for (int jj = 0; jj < S; ++jj) {
          const uint32_t src = map_shared_rank(smem_u32(red + (jj * BM + i) * rs + c), t);
          const float4 a = ld_shared_cluster_f32x4(src), b = ld_shared_cluster_f32x4(src + 16);
          const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] = __fadd_rn(acc[e], v[e]);
        }
      }
      if (m0 + i < p.M) {
        // hi = bf16(acc), lo = bf16(acc - hi): hi + lo carries acc to ~2^-17
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          hi[e] = pack_bf16x2(acc[2 * e], acc[2 * e + 1]);
          lo[e] = pack_bf16x2(acc[2 * e] - bf16_lo(hi[e]), acc[2 * e + 1] - bf16_hi(hi[e]));
        }
        __nv_bfloat16* dst = p.xl1 + static_cast<size_t>(m0 + i) * (2 * p.r_pad) + c;
        *reinterpret_cast<uint4*>(dst) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(dst + p.r_pad) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    }
  }
  // no CTA leaves while a peer may still read its shared memory
  if (p.C > 1) cluster_sync();
  if (warp == 1 && has_lr) {
    // every MMA this CTA issued has retired before its TMEM is released
    mbar_wait(acc_full, 0, drain_budget(p.budget), nullptr);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

// W8A8 per-token scale (SVDQuant paper, Sec. 5.1, 8-bit setting):
// s_x[m] = max_k |fp32(x[m,k]) * (1/lambda_k)| / 127, IEEE fp32, one warp per
// row.  Each lane keeps four 16-byte loads of the row in flight; the guards
// keep every load inside the row.
__global__ void w8_row_scale_kernel(const __nv_bfloat16* __restrict__ X, const float* __restrict__ inv_lambda,
                                    int M, int K, float* __restrict__ sx) {
  const int m = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  griddep_launch_dependents();
  griddep_wait();
  if (m >= M) return;
  const uint4* xr = reinterpret_cast<const uint4*>(X + static_cast<size_t>(m) * K);
  const float4* il = reinterpret_cast<const float4*>(inv_lambda);
  const int n8 = K / 8;   // 16-byte chunks of the row
  float amax[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int c0 = lane; c0 < n8; c0 += 4 * 32) {
    uint4 raw[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = c0 + 32 * u;
      raw[u] = c < n8 ? __ldg(xr + c) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = c0 + 32 * u;
      if (c < n8) {
        const float4 l0 = __ldg(il + 2 * c), l1 = __ldg(il + 2 * c + 1);
        float a = amax[u];
        a = fmax3(a, fabsf(__fmul_rn(bf16_lo(raw[u].x), l0.x)), fabsf(__fmul_rn(bf16_hi(raw[u].x), l0.y)));
        a = fmax3(a, fabsf(__fmul_rn(bf16_lo(raw[u].y), l0.z)), fabsf(__fmul_rn(bf16_hi(raw[u].y), l0.w)));
        a = fmax3(a, fabsf(__fmul_rn(bf16_lo(raw[u].z), l1.x)), fabsf(__fmul_rn(bf16_hi(raw[u].z), l1.y)));
        a = fmax3(a, fabsf(__fmul_rn(bf16_lo(raw[u].w), l1.z)), fabsf(__fmul_rn(bf16_hi(raw[u].w), l1.w)));
        amax[u] = a;
      }
    }
  }
  float a = fmaxf(fmaxf(amax[0], amax[1]), fmaxf(amax[2], amax[3]));
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if (lane == 0) sx[m] = __fdiv_rn(a, 127.0f);
}

}  // namespace svdq
