// gemm_int4.cuh -- the INT4 (groups of 64, fp16 scales) variant of the fused
// 4-bit GEMM + low-rank up-projection + bias.
//
// SVDQuant Sec. 5.1: INT4 quantization uses groups of 64 with 16-bit scales.
// Per-group scales s_x[m,g] s_w[g,n] do not factor out of a K sum, so each
// 64-wide group is one tcgen05 kind::i8 product (two K = 32 MMAs) into one of
// four TMEM partial buffers; sixteen drain warps scale every partial and
// accumulate it in fp32 registers while the tensor core fills the other
// buffers.  The low-rank tail (kind::f16, fp32) goes through the same buffers
// with scale 1.
//
// Weight codes stay at 4 bits in HBM (N x K/2 bytes, element 2i in the low
// nibble, two's complement).  The drain warps also unpack each stage's packed
// B tile in shared memory, a few stages ahead of the MMA: every nibble goes to
// the high half of its own byte, so the int8 the tensor core reads is 16 q
// (the sign comes along for free, three integer operations per eight codes),
// and within each run of eight values the bytes come out in the K order
// 0 2 4 6 1 3 5 7.  The activation codes (int8, written by the activation
// kernel) are stored in that same order, so every product q_x q_w meets its
// partner and the group's integer sum is 16 P with P = sum q_x q_w.
//
// The partial reaches the drain already as fp32: each buffer is pre-filled
// with the bit pattern of 1.5 * 2^23 and the MMAs accumulate onto it, so the
// bits read back are those of v = 1.5 * 2^23 + 16 P exactly (|16 P| <= 16 * 64
// * 49 < 2^22).  After reading a buffer the drain refills it.  Per output and
// group the drain then issues two fused multiply-adds, on packed pairs:
//   t   = v * (s_w / 16) + c,   c = -1.5 * 2^19 * s_w     (t = P s_w exactly:
//         P s_w has at most 23 significant bits, and c is exact)
//   acc = t * s_x + acc
// with (s_w / 16, c) prepared per weight column beside the fp16 scales.
//
//   warp 0     : TMA producer (A 128 x 64 int8, the packed B 128 x 32 bytes,
//                the group's activation scales (fp16) and the weight columns'
//                (s_w / 16, c) pairs; then the XL1 / L2^T chunks of the tail)
//   warp 1     : TMEM owner, MMA issuer
//   warps 2-17 : unpack of B (each a 16th of the tile, kI4Ahead stages ahead)
//                and drain + epilogue: warp w serves TMEM lane quarter w % 4
//                and output columns [32 ((w - 2) / 4), +32) of the 128 x 128
//                tile.  Four warps per scheduler hide the TMEM load latency.
#pragma once

#include "gemm_nvfp4.cuh"
#include "svdq_formats.cuh"
#include "svdq_ptx.cuh"

namespace svdq {

constexpr int kI4BM = 128;
constexpr int kI4BN = 128;
constexpr int kI4BK = 64;                 // one group
constexpr int kI4EpiWarps = 16;
constexpr int kI4Threads = 32 * (2 + kI4EpiWarps);
constexpr int kI4Bufs = 4;                // TMEM partial buffers of kI4BN columns
constexpr int kI4Ahead = 2;               // stages the unpack runs ahead of the drain
constexpr uint32_t kI4AOff = 0;                            // 128 x 64 B (int8 codes or a tail chunk)
constexpr uint32_t kI4BOff = kI4BM * 64;                   // 8192: unpacked B, 128 x 64 B
constexpr uint32_t kI4BpOff = kI4BOff + kI4BN * 64;        // 16384: packed B, 128 x 32 B
constexpr uint32_t kI4SxOff = kI4BpOff + kI4BN * 32;       // 20480: activation scales, 128 fp16
constexpr uint32_t kI4SwOff = kI4SxOff + kI4BM * 2;        // 20736: 64 (s_w / 16, c) column pairs
constexpr uint32_t kI4StageBytes = 22528;                  // 22 KB, multiple of 1024
constexpr int kI4Stages = 9;
constexpr uint32_t kI4BarBytes = 512;                      // 3 S + 2 NB + 1 mbarriers, TMEM address, flag
constexpr uint32_t kI4SmemBytes = kI4StageBytes * kI4Stages + kI4BarBytes + 1024;
constexpr uint32_t kI4Magic = 0x4B400000u;                 // bits of 1.5 * 2^23
static_assert(kI4SwOff + 64 * 16 <= kI4StageBytes, "stage layout");
static_assert(kI4Stages >= kI4Ahead + 2, "the unpack look-ahead needs free stages");
static_assert((3 * kI4Stages + 2 * kI4Bufs + 1) * 8 + 8 <= kI4BarBytes, "barrier area");

// Low-rank tail chunks of at most 32 bf16 columns (64-byte rows: they fit the
// A and B regions of a stage).
__host__ __device__ inline int i4_lr_chunk_cols(int k_tail) { return k_tail < 32 ? k_tail : 32; }
__host__ __device__ inline int i4_lr_num_chunks(int k_tail) {
  return k_tail == 0 ? 0 : (k_tail + 31) / 32;
}

struct GemmI4Params {
  int M, N, K;
  int groups;          // K / 64
  int m_tiles, n_tiles, num_tiles;
  int group_m;         // tile order (gemm_tile_coords)
  int r_tail;          // tail K: 2 r_pad (X_hat L1 as hi | lo against L2^T | L2^T), 0 = none
  const uint16_t* sx;  // fp16 [K/64][M_pad]
  const float4* swc;   // [K/64][N_pad/2]: (s_w[2i] / 16, s_w[2i+1] / 16, c[2i], c[2i+1])
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

__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b,
                                                     unsigned long long c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

__device__ __forceinline__ unsigned long long f2_add(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// Eight packed two's-complement codes (element 2i in the low nibble of byte
// i) -> eight int8 values 16 q, K order 0 2 4 6 | 1 3 5 7.
__device__ __forceinline__ uint2 i4_unpack8(uint32_t w) {
  return make_uint2((w << 4) & 0xF0F0F0F0u, w & 0xF0F0F0F0u);
}

// One drain warp's share of unpacking step u: wait for the stage's copies,
// turn 8 packed bytes (16 codes) of B into the MMA layout (64-byte rows,
// 64-byte swizzle: 16-byte chunk c of row r at c ^ ((r >> 1) & 3)), and
// arrive on the stage's `unpacked` barrier.  Tail steps only arrive.
__device__ __forceinline__ void i4_unpack_step(int u, uint8_t* smem, uint64_t* full, uint64_t* unpacked,
                                               int steps_per_tile, int groups, uint32_t u_src, uint32_t u_dst,
                                               long long budget, volatile int* abort_flag, bool& ok,
                                               uint32_t lane) {
  const int s = u % kI4Stages;
  if (ok && !warp_wait(&full[s], (u / kI4Stages) & 1, budget, abort_flag)) {
    if (lane == 0) raise_error(kErrWaitGemm);
    *abort_flag = 1;
    ok = false;
  }
  if (ok && (u % steps_per_tile) < groups) {
    uint8_t* st = smem + s * kI4StageBytes;
    const uint2 w = *reinterpret_cast<const uint2*>(st + u_src);
    const uint2 a = i4_unpack8(w.x), b = i4_unpack8(w.y);
    *reinterpret_cast<uint4*>(st + u_dst) = make_uint4(a.x, a.y, b.x, b.y);
    fence_proxy_async_smem();
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(&unpacked[s]);
}

__global__ void __launch_bounds__(kI4Threads, 1)
    gemm_int4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_bp,
                     const __grid_constant__ CUtensorMap tm_xl1,
                     const __grid_constant__ CUtensorMap tm_l2t, const GemmI4Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  constexpr int S = kI4Stages;
  constexpr int NB = kI4Bufs;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kI4StageBytes * S);
  uint64_t* unpacked = full + S;    // [S]: B of the stage is in its MMA layout
  uint64_t* empty = unpacked + S;
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
  // steps this CTA runs over all its tiles (every role walks the same sequence)
  const int my_tiles = p.num_tiles > static_cast<int>(blockIdx.x)
                           ? (p.num_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                                 static_cast<int>(gridDim.x)
                           : 0;
  const int total_steps = my_tiles * steps_per_tile;

  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&unpacked[s], kI4EpiWarps);
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
      tmem_st32_const(tmem_base + ((q * 32u) << 16) + kI4BN * b + 32u * h, kI4Magic);
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();   // the activation codes, scales and XL1 come from the previous kernel

  if (warp == 0) {
    if (elect_one()) {
      prefetch_tmap(&tm_a);
      prefetch_tmap(&tm_bp);
      if (n_lr) {
        prefetch_tmap(&tm_xl1);
        prefetch_tmap(&tm_l2t);
      }
      const uint32_t main_tx = kI4BM * 64 + kI4BN * 32 + kI4BM * 2 + (kI4BN / 2) * 16;
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
            tma_load_2d(st + kI4BpOff, &tm_bp, &full[s], g * (kI4BK / 2), n0);
            bulk_load(st + kI4SxOff, p.sx + static_cast<size_t>(g) * p.M_pad + m0, kI4BM * 2, &full[s]);
            bulk_load(st + kI4SwOff, p.swc + static_cast<size_t>(g) * (p.N_pad / 2) + n0 / 2, (kI4BN / 2) * 16,
                      &full[s]);
          } else {
            const int c = step - p.groups;
            mbar_arrive_expect_tx(&full[s], lr_tx);
            tma_load_2d(st + kI4AOff, &tm_xl1, &full[s], c * 32, m0);
            tma_load_2d(st + kI4BOff, &tm_l2t, &full[s], c * 32, n0);
          }
        }
      }
      // never leave while a copy into this CTA's shared memory is still in flight
      // (whether or not a wait ran out, and in whichever role)
      for (int i = (it > S ? it - S : 0); i < it; ++i)
        mbar_wait(&full[i % S], (i / S) & 1, drain_budget(p.budget), nullptr);
    }
  } else if (warp == 1) {
    if (elect_one()) {
      const uint32_t idesc_main = idesc_s8_s32(kI4BM, kI4BN);
      const uint32_t idesc_lr = idesc_bf16_f32(kI4BM, kI4BN);
      const uint32_t lr_row_bytes = static_cast<uint32_t>(lr_cols) * 2;
      for (int it = 0; it < total_steps; ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        const int b = it % NB;
        const uint32_t pph = (it / NB) & 1;
        const bool tail = (it % steps_per_tile) >= p.groups;
        if (!mbar_wait(&pempty[b], pph ^ 1, p.budget, abort_flag) ||
            !mbar_wait(&full[s], ph, p.budget, abort_flag) ||
            !mbar_wait(&unpacked[s], ph, p.budget, abort_flag)) {
          raise_error(kErrWaitGemm);
          *abort_flag = 1;
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
            mma_i8(d, make_kmajor_desc(a0 + 32 * j, 64), make_kmajor_desc(b0 + 32 * j, 64), idesc_main, 1u);
        } else {
          for (int j = 0; j < lr_cols / 16; ++j)
            mma_bf16(d, make_kmajor_desc(a0 + 32 * j, lr_row_bytes), make_kmajor_desc(b0 + 32 * j, lr_row_bytes),
                     idesc_lr, j > 0 ? 1u : 0u);
        }
        tc_commit(&empty[s]);
        tc_commit(&pfull[b]);
      }
      tc_commit(mma_done);
    }
  } else {
    // ------------------------------------------------ unpack + drain / epilogue
    const uint32_t d = warp - 2;               // 0 .. 15
    const uint32_t q = warp & 3u;              // TMEM lane quarter this warp may access
    const uint32_t h = d >> 2;                 // 32-column slice of the tile
    const uint32_t row = q * 32 + lane;
    // unpack share: 8 packed bytes (16 codes) of B row ur, quarter uq
    const uint32_t ut = d * 32 + lane;         // 0 .. 511
    const uint32_t ur = ut >> 2, uq = ut & 3u;
    const uint32_t u_src = kI4BpOff + ur * 32 + uq * 8;
    const uint32_t u_dst = kI4BOff + ur * 64 + ((uq ^ ((ur >> 1) & 3u)) << 4);   // 64-byte swizzle
    bool ok = true;

    for (int u = 0; u < kI4Ahead && u < total_steps; ++u)
      i4_unpack_step(u, smem, full, unpacked, steps_per_tile, p.groups, u_src, u_dst, p.budget, abort_flag, ok, lane);
    int it = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      int m_blk, n_blk;
      gemm_tile_coords(p.m_tiles, p.n_tiles, p.group_m, tile, m_blk, n_blk);
      const int m = m_blk * kI4BM + static_cast<int>(row);
      unsigned long long acc[16];   // 32 fp32 accumulators, pairs of adjacent columns
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[j] = 0ull;
      for (int step = 0; step < steps_per_tile; ++step, ++it) {
        if (it + kI4Ahead < total_steps)
          i4_unpack_step(it + kI4Ahead, smem, full, unpacked, steps_per_tile, p.groups, u_src, u_dst, p.budget,
                         abort_flag, ok, lane);
        const int s = it % S;
        const int b = it % NB;
        const uint32_t pph = (it / NB) & 1;
        if (ok && !warp_wait(&pfull[b], pph, p.budget, abort_flag)) {
          if (lane == 0) raise_error(kErrWaitGemm);
          *abort_flag = 1;
          ok = false;
        }
        if (ok) {
          tc_fence_after();
          const uint8_t* st = smem + s * kI4StageBytes;
          const uint32_t taddr = tmem_base + ((q * 32u) << 16) + kI4BN * b + 32u * h;
          const bool main_step = step < p.groups;
          unsigned long long sx2 = 0ull;
          if (main_step) {
            const float sx = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(st + kI4SxOff)[row]));
            sx2 = f2_pack(sx, sx);
          }
          const ulonglong2* swc = reinterpret_cast<const ulonglong2*>(st + kI4SwOff) + 16 * h;
          // two halves of 16 columns (16 loaded values live at a time)
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t r[16];
            tmem_ld16(taddr + 16u * half, r);
            tmem_wait_ld();
            if (main_step) {
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const ulonglong2 wc = swc[8 * half + j];   // (s_w / 16, c) of columns 32 h + 16 half + 2 j, + 1
                acc[8 * half + j] =
                    f2_fma(f2_fma(u2_pack(r[2 * j], r[2 * j + 1]), wc.x, wc.y), sx2, acc[8 * half + j]);
              }
            } else {
#pragma unroll
              for (int j = 0; j < 8; ++j) acc[8 * half + j] = f2_add(acc[8 * half + j], u2_pack(r[2 * j], r[2 * j + 1]));
            }
          }
          tmem_st32_const(taddr, kI4Magic);   // the buffer holds the offset again
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&pempty[b]);
          mbar_arrive(&empty[s]);    // done with this stage's scales
        }
      }
      if (!ok) continue;   // keep walking the steps so the barriers stay matched
      // bias, bf16, store: 32 columns of this row
      const int n_base = n_blk * kI4BN + 32 * static_cast<int>(h);
      if (m < p.M) {
        __nv_bfloat16* yrow = p.Y + static_cast<size_t>(m) * p.N;
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
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
    mbar_wait(mma_done, 0, drain_budget(p.budget), nullptr);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace svdq
