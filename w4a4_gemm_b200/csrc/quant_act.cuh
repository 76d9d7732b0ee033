// quant_act.cuh -- the fused activation kernel: smoothing, per-group 4-bit
// quantization and the low-rank down-projection in one pass over X.
//
// SVDQuant Sec. 4.3 (Nunchaku, Fig. 6b): the down-projection X_hat L1 shares
// its input with the quantizer, so both are computed from one read of X.
//
// CTA = 128 rows x a contiguous range of 64-wide K tiles.  Row blocks with
// too few CTAs to fill the GPU are split along K across a thread-block
// cluster; the rank-r partial products are then summed in fixed rank order
// through distributed shared memory.
//   warp 0      : TMA producer (X tile 128x64 bf16, L1^T tile r_pad x 64, 1/lambda)
//   warp 1      : TMEM owner; one lane issues the tcgen05 bf16 MMAs
//                 XL1 += bf16(x_hat) (128 x 64) * L1^T(64 x r_pad)
//   warps 2..9  : quantizers; warp w serves TMEM lane quarter w % 4 (rows)
//                 and K half (w - 2) / 4 of every tile.  They smooth X,
//                 quantize it, store codes and scales, and write bf16(x_hat)
//                 back in place as the MMA's A operand.
#pragma once

#include "svdq_formats.cuh"
#include "svdq_ptx.cuh"

namespace svdq {

constexpr int kQuantBM = 128;
constexpr int kQuantBK = 64;
constexpr int kQuantStages = 4;
constexpr int kQuantThreads = 320;
constexpr int kQuantWarps = 8;  // quantizer warps

struct QuantParams {
  int M, K;
  int r_pad;        // 0 = no low-rank branch; else 16, 32, 64, 128, 192 or 256
  int kt_total;     // K / 64
  int ksplit;       // CTAs per 128-row block (cluster extent along y)
  int M_pad;        // M rounded up to 128
  int sf_kcols;     // NVFP4: K_pad / 64 scale atoms per 128-row block
  const float* inv_lambda;
  uint8_t* codes;   // NVFP4: M x K/2 packed E2M1; INT4: M x K int8
  uint8_t* sf;      // NVFP4: 512-byte atoms; INT4: fp16 [K/64][M_pad]
  __nv_bfloat16* xl1;  // M x r_pad
  long long budget;
};

struct QuantSmem {
  uint32_t x_off, l1_off, il_off, stage_bytes, red_off, bar_off, total;
};

__host__ __device__ inline QuantSmem quant_smem_layout(int r_pad) {
  QuantSmem L;
  L.x_off = 0;
  L.l1_off = kQuantBM * kQuantBK * 2;                      // 16384
  L.il_off = L.l1_off + r_pad * 128;
  uint32_t sb = L.il_off + kQuantBK * 4;
  L.stage_bytes = (sb + 1023u) & ~1023u;
  // the K-split partial sums reuse the stage buffers once the K loop is over
  // (128 x r_pad fp32 never exceeds the four stages)
  L.red_off = 0;
  L.bar_off = L.stage_bytes * kQuantStages;
  L.total = L.bar_off + 256 + 1024;                        // barriers + alignment slack
  return L;
}

template <int FMT>  // 0 = NVFP4 (groups of 16), 1 = INT4 (groups of 64)
__global__ void __launch_bounds__(kQuantThreads, 1)
    quant_act_kernel(const __grid_constant__ CUtensorMap tm_x,
                     const __grid_constant__ CUtensorMap tm_l1t, const QuantParams p) {
  extern __shared__ uint8_t smem_raw[];
  const QuantSmem L = quant_smem_layout(p.r_pad);
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* xready = full + kQuantStages;
  uint64_t* empty = xready + kQuantStages;
  uint64_t* acc_full = empty + kQuantStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const bool has_lr = p.r_pad > 0;
  const int m_blk = blockIdx.x;
  const int m0 = m_blk * kQuantBM;
  const int ks = blockIdx.y;
  const int kt_begin = (ks * p.kt_total) / p.ksplit;
  const int kt_end = ((ks + 1) * p.kt_total) / p.ksplit;
  const int nkt = kt_end - kt_begin;
  const uint32_t tmem_cols = p.r_pad <= 32 ? 32u : (p.r_pad <= 64 ? 64u : (p.r_pad <= 128 ? 128u : 256u));

  if (threadIdx.x == 0) {
    for (int s = 0; s < kQuantStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&xready[s], kQuantWarps);
      mbar_init(&empty[s], has_lr ? 1 : kQuantWarps);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1 && has_lr) {
    tmem_alloc(tmem_holder, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = has_lr ? *tmem_holder : 0u;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      prefetch_tmap(&tm_x);
      if (has_lr) prefetch_tmap(&tm_l1t);
      const uint32_t tx = kQuantBM * kQuantBK * 2 + (has_lr ? p.r_pad * 128 : 0) + kQuantBK * 4;
      int issued = 0;
      for (int i = 0; i < nkt; ++i) {
        const int s = i % kQuantStages;
        const uint32_t ph = (i / kQuantStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, p.budget, abort_flag)) {
          raise_error(kErrWaitQuant);
          *abort_flag = 1;
          break;
        }
        uint8_t* st = smem + s * L.stage_bytes;
        const int kt = kt_begin + i;
        mbar_arrive_expect_tx(&full[s], tx);
        tma_load_2d(st + L.x_off, &tm_x, &full[s], kt * kQuantBK, m0);
        if (has_lr) tma_load_2d(st + L.l1_off, &tm_l1t, &full[s], kt * kQuantBK, 0);
        bulk_load(st + L.il_off, p.inv_lambda + kt * kQuantBK, kQuantBK * 4, &full[s]);
        issued = i + 1;
      }
      // never leave while a copy into this CTA's shared memory is still in flight
      if (*abort_flag) {
        for (int i = (issued > kQuantStages ? issued - kQuantStages : 0); i < issued; ++i)
          mbar_wait(&full[i % kQuantStages], (i / kQuantStages) & 1, p.budget, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (has_lr && elect_one()) {
      const uint32_t idesc = idesc_bf16_f32(kQuantBM, p.r_pad);
      bool ok = true;
      for (int i = 0; i < nkt; ++i) {
        const int s = i % kQuantStages;
        const uint32_t ph = (i / kQuantStages) & 1;
        if (!mbar_wait(&xready[s], ph, p.budget, abort_flag)) {
          raise_error(kErrWaitQuant);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + s * L.stage_bytes + L.x_off);
        const uint32_t b0 = smem_u32(smem + s * L.stage_bytes + L.l1_off);
#pragma unroll
        for (int k = 0; k < kQuantBK / 16; ++k) {
          mma_bf16(tmem_base, make_kmajor_desc(a0 + 32 * k, 128), make_kmajor_desc(b0 + 32 * k, 128),
                   idesc, (i > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(&empty[s]);
      }
      (void)ok;
      tc_commit(acc_full);  // also covers an early exit: waits for every issued MMA
    }
  } else {
    // ------------------------------------------------------------ quantizers
    // NVFP4: warp half h quantizes K columns [32h, 32h + 32) of every tile (two
    // groups of 16).  INT4: a group spans the whole 64-wide tile, so the h = 0
    // warps quantize it alone and the h = 1 warps only take part in the
    // hand-off to the MMA.
    const uint32_t q = warp & 3u;             // TMEM lane quarter = row group
    const uint32_t h = (warp - 2) >> 2;       // K half of each 64-wide tile
    const uint32_t row = q * 32 + lane;
    const int m = m0 + static_cast<int>(row);
    const bool row_ok = m < p.M;
    constexpr int kChunks = FMT == 0 ? 4 : 8;   // 16-byte chunks (8 bf16) per thread
    const bool active = FMT == 0 || h == 0;
    const uint32_t c0 = FMT == 0 ? 4 * h : 0;
    for (int i = 0; i < nkt; ++i) {
      const int s = i % kQuantStages;
      const uint32_t ph = (i / kQuantStages) & 1;
      if (!warp_wait(&full[s], ph, p.budget, abort_flag)) {
        if (lane == 0) raise_error(kErrWaitQuant);
        *abort_flag = 1;
        break;
      }
      if (active) {
        uint8_t* st = smem + s * L.stage_bytes;
        const float* il = reinterpret_cast<const float*>(st + L.il_off) + 8 * c0;
        uint8_t* xrow = st + L.x_off + row * 128;
        const int kt = kt_begin + i;
        float v[8 * kChunks];
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          const uint32_t chunk = ((c0 + c) ^ (row & 7u)) << 4;   // 128-byte swizzle
          const uint4 raw = *reinterpret_cast<const uint4*>(xrow + chunk);
          const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            v[8 * c + 2 * j] = __fmul_rn(bf16_lo(w4[j]), il[8 * c + 2 * j]);
            v[8 * c + 2 * j + 1] = __fmul_rn(bf16_hi(w4[j]), il[8 * c + 2 * j + 1]);
          }
        }
        if constexpr (FMT == 0) {
          uint32_t cw[4];
          const uint32_t s0 = quant16_nvfp4(v, cw);
          const uint32_t s1 = quant16_nvfp4(v + 16, cw + 2);
          if (row_ok) {
            uint8_t* dst = p.codes + static_cast<size_t>(m) * (p.K / 2) + kt * (kQuantBK / 2) + 16 * h;
            *reinterpret_cast<uint4*>(dst) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
          }
          // scale atom: 128 rows x 4 scales, byte (row % 32) * 16 + (row / 32) * 4 + k4
          uint8_t* atom = p.sf + (static_cast<size_t>(m_blk) * p.sf_kcols + kt) * 512;
          *reinterpret_cast<uint16_t*>(atom + (row & 31u) * 16 + (row >> 5) * 4 + 2 * h) =
              static_cast<uint16_t>(row_ok ? (s0 | (s1 << 8)) : 0u);
        } else {
          float amax = 0.0f;
#pragma unroll
          for (int j = 0; j < 64; ++j) amax = fmaxf(amax, fabsf(v[j]));
          const uint16_t sh = int4_scale_bits(amax);
          const float sd = __half2float(__ushort_as_half(sh));
          uint32_t packed[16];
          if (sd == 0.0f) {
#pragma unroll
            for (int j = 0; j < 16; ++j) packed[j] = 0u;
          } else {
            const float inv = __frcp_rn(sd);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              uint32_t w = 0;
#pragma unroll
              for (int b = 0; b < 4; ++b)
                w |= (static_cast<uint32_t>(int4_code(v[4 * j + b], inv)) & 0xFFu) << (8 * b);
              packed[j] = w;
            }
          }
          if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(p.codes + static_cast<size_t>(m) * p.K + kt * kQuantBK);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
          }
          reinterpret_cast<uint16_t*>(p.sf)[static_cast<size_t>(kt) * p.M_pad + m0 + row] =
              row_ok ? sh : static_cast<uint16_t>(0);
        }
        if (has_lr) {
          // bf16(x_hat) back into the tile at the same swizzled positions: the MMA's A operand
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
            const uint32_t chunk = ((c0 + c) ^ (row & 7u)) << 4;
            uint4 o;
            o.x = pack_bf16x2(v[8 * c + 0], v[8 * c + 1]);
            o.y = pack_bf16x2(v[8 * c + 2], v[8 * c + 3]);
            o.z = pack_bf16x2(v[8 * c + 4], v[8 * c + 5]);
            o.w = pack_bf16x2(v[8 * c + 6], v[8 * c + 7]);
            *reinterpret_cast<uint4*>(xrow + chunk) = o;
          }
          fence_proxy_async_smem();
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(has_lr ? &xready[s] : &empty[s]);
    }
  }

  __syncwarp();

  // ---------------------------------------------------------------- XL1 out
  float* red = reinterpret_cast<float*>(smem + L.red_off);
  const bool epi = has_lr && warp >= 2 && warp < 6;
  if (epi) {
    const uint32_t q = warp & 3u;
    const uint32_t row = q * 32 + lane;
    const bool got = warp_wait(acc_full, 0, p.budget, abort_flag);
    if (!got) {
      if (lane == 0) raise_error(kErrWaitQuant);
      *abort_flag = 1;
    }
    tc_fence_after();
    for (int c = 0; c < p.r_pad; c += 16) {
      uint32_t r[16];
      tmem_ld16(tmem_base + ((q * 32u) << 16) + c, r);
      tmem_wait_ld();
      if (p.ksplit == 1) {
        const int m = m0 + static_cast<int>(row);
        if (m < p.M) {
          uint4 o0, o1;
          o0.x = pack_bf16x2(__uint_as_float(r[0]), __uint_as_float(r[1]));
          o0.y = pack_bf16x2(__uint_as_float(r[2]), __uint_as_float(r[3]));
          o0.z = pack_bf16x2(__uint_as_float(r[4]), __uint_as_float(r[5]));
          o0.w = pack_bf16x2(__uint_as_float(r[6]), __uint_as_float(r[7]));
          o1.x = pack_bf16x2(__uint_as_float(r[8]), __uint_as_float(r[9]));
          o1.y = pack_bf16x2(__uint_as_float(r[10]), __uint_as_float(r[11]));
          o1.z = pack_bf16x2(__uint_as_float(r[12]), __uint_as_float(r[13]));
          o1.w = pack_bf16x2(__uint_as_float(r[14]), __uint_as_float(r[15]));
          uint4* dst = reinterpret_cast<uint4*>(p.xl1 + static_cast<size_t>(m) * p.r_pad + c);
          dst[0] = o0;
          dst[1] = o1;
        }
      } else {
        float* dst = red + row * p.r_pad + c;
#pragma unroll
        for (int j = 0; j < 16; j += 4)
          *reinterpret_cast<float4*>(dst + j) =
              make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                          __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
      }
    }
  }
  if (has_lr && p.ksplit > 1) {
    cluster_sync();  // every partial is in its CTA's shared memory
    if (ks == 0 && epi) {
      const uint32_t row = (warp & 3u) * 32 + lane;
      const int m = m0 + static_cast<int>(row);
      const uint32_t base = smem_u32(red + row * p.r_pad);
      for (int c = 0; c < p.r_pad; c += 8) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int rk = 0; rk < p.ksplit; ++rk) {
          const uint32_t a = map_shared_rank(base + 4 * c, rk);
          const float4 x0 = ld_shared_cluster_f32x4(a);
          const float4 x1 = ld_shared_cluster_f32x4(a + 16);
          acc[0] += x0.x; acc[1] += x0.y; acc[2] += x0.z; acc[3] += x0.w;
          acc[4] += x1.x; acc[5] += x1.y; acc[6] += x1.z; acc[7] += x1.w;
        }
        if (m < p.M) {
          uint4 o;
          o.x = pack_bf16x2(acc[0], acc[1]);
          o.y = pack_bf16x2(acc[2], acc[3]);
          o.z = pack_bf16x2(acc[4], acc[5]);
          o.w = pack_bf16x2(acc[6], acc[7]);
          *reinterpret_cast<uint4*>(p.xl1 + static_cast<size_t>(m) * p.r_pad + c) = o;
        }
      }
    }
    cluster_sync();  // keep every CTA's partial alive until rank 0 has read it
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1 && has_lr) {
    // every MMA this CTA issued has retired before its TMEM is released
    mbar_wait(acc_full, 0, p.budget, nullptr);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

}  // namespace svdq
