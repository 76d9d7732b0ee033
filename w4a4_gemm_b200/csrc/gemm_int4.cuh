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
// nibble, two's complement).  Two unpack warps turn each stage's packed B tile
// into the MMA's int8 layout in shared memory as soon as it lands: every
// nibble goes to the high half of its own byte, so the int8 the tensor core
// reads is 16 q (the sign comes along for free, three integer operations per
// eight codes), and within each run of eight values the bytes come out in the
// K order 0 2 4 6 1 3 5 7.  The activation codes (int8, written by the
// activation kernel) are stored in that same order, so every product q_x q_w
// meets its partner and the group's integer sum is 16 P, P = sum q_x q_w.
//
// The partial reaches the drain already as an fp32 value: before a group's two
// int8 MMAs the MMA issuer writes 1.5 * 2^23 into the partial buffer with one
// bf16 MMA of two constant tiles (A rows (1, 0, ...), B rows (1.5 * 2^23, 0,
// ...), accumulate off); the int8 MMAs accumulate onto that offset's bits, which
// are then the bits of the fp32 value 1.5 * 2^23 + 16 P (|16 P| <= 16 * 64 * 49
// < 2^22); a second bf16 MMA (B rows -1.5 * 2^23, accumulate on) subtracts the
// offset in fp32, exactly, leaving 16 P.  The drain only reads TMEM, and per
// output pair and group issues two packed fp32 operations:
//   s   = s_x * (s_w / 16)   (exact: two fp16 values and a power of two)
//   acc = 16 P * s + acc     (one rounding)
// with s_w / 16 prepared per weight column beside the fp16 scales.
//
//   warp 0      : TMA producer (A 128 x 64 int8, the packed B 128 x 32 bytes,
//                 the group's activation scales (fp16) and the weight columns'
//                 s_w / 16; then the XL1 / L2^T chunks of the tail)
//   warp 1      : TMEM owner, MMA issuer
//   warps 2-9   : drain + epilogue: warp w serves TMEM lane quarter w % 4 and
//                 output columns [64 ((w - 2) / 4), +64) of the 128 x 128 tile,
//                 read from TMEM with one 64-column load per group
//   warps 10-11 : unpack of the packed B tiles, stage by stage as they land
#pragma once

#include "gemm_nvfp4.cuh"
#include "svdq_formats.cuh"
#include "svdq_ptx.cuh"

namespace svdq {

constexpr int kI4BM = 128;
constexpr int kI4BN = 128;
constexpr int kI4BK = 64;                 // one group
constexpr int kI4EpiWarps = 8;
constexpr int kI4UnpackWarps = 2;
constexpr int kI4Threads = 32 * (2 + kI4EpiWarps + kI4UnpackWarps);
constexpr int kI4Bufs = 4;                // TMEM partial buffers of kI4BN columns
constexpr uint32_t kI4AOff = 0;                            // 128 x 64 B (int8 codes or a tail chunk)
constexpr uint32_t kI4BOff = kI4BM * 128;                  // 16384
constexpr uint32_t kI4BpOff = kI4BOff + kI4BN * 128;       // 32768
constexpr uint32_t kI4SxOff = kI4BpOff + kI4BN * 32;       // 20480: activation scales, 128 fp16
constexpr uint32_t kI4SwOff = kI4SxOff + kI4BM * 2;        // s_w / 16 of the tile's 128 columns
constexpr uint32_t kI4StageBytes = 38912;
constexpr int kI4Stages = 5;
constexpr uint32_t kI4ConstOff = kI4StageBytes * kI4Stages;  // the offset MMAs' constant 128 x 16 bf16 tiles:
                                                             // A = (1, 0, ...), B = (+-1.5 * 2^23, 0, ...)
constexpr uint32_t kI4BarBytes = 512;                      // 3 S + 2 NB + 1 mbarriers, TMEM address, flag
constexpr uint32_t kI4SmemBytes = kI4ConstOff + 12288 + kI4BarBytes + 1024;
static_assert(kI4SwOff + kI4BN * 4 <= kI4StageBytes, "stage layout");
static_assert((3 * kI4Stages + 2 * kI4Bufs + 1) * 8 + 8 <= kI4BarBytes, "barrier area");

// Low-rank tail chunks of at most 64 bf16 columns (128-byte rows: 128 of them
// fill the 16 KB A and B regions of a stage).
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
  const float* sw16;   // [K/64][N_pad]: s_w / 16 (exact)
  int M_pad, N_pad;
  const __nv_bfloat16* bias;
  __nv_bfloat16* Y;
  long long budget;
};

// 64 consecutive 32-bit TMEM columns of this warp's 32 lanes into 64 registers.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
      "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
      "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
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

// Eight packed two's-complement codes (element 2i in the low nibble of byte
// i) -> eight int8 values 16 q, K order 0 2 4 6 | 1 3 5 7.
__device__ __forceinline__ uint2 i4_unpack8(uint32_t w) {
  return make_uint2((w << 4) & 0xF0F0F0F0u, w & 0xF0F0F0F0u);
}

__global__ void __launch_bounds__(kI4Threads, 1)
    gemm_int4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_bp,
                     const __grid_constant__ CUtensorMap tm_xl1,
                     const __grid_constant__ CUtensorMap tm_l2t, const GemmI4Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  constexpr int S = kI4Stages;
  constexpr int NB = kI4Bufs;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kI4ConstOff + 12288);
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
      mbar_init(&unpacked[s], kI4UnpackWarps);
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
  if (threadIdx.x < 384) {
    // The offset MMAs' operands, 128 x 16 bf16 each, K-major, 32-byte swizzle
    // (16-byte chunk c of row r at c ^ ((r >> 2) & 1)): A rows (1, 0, ..., 0),
    // B rows (1.5 * 2^23, 0, ..., 0) and (-1.5 * 2^23, 0, ..., 0), so that
    // D = A B^T is +-1.5 * 2^23 in every element, exactly.
    const uint32_t t = threadIdx.x & 127u, which = threadIdx.x >> 7;
    uint8_t* rowp = smem + kI4ConstOff + which * 4096u + t * 32;
    const uint32_t first = which == 0 ? 0x3F80u : (which == 1 ? 0x4B40u : 0xCB40u);   // 1.0, +-1.5 * 2^23
    const uint32_t c0 = (t >> 2) & 1u;                              // physical chunk of k = 0 .. 7
    *reinterpret_cast<uint4*>(rowp + (c0 << 4)) = make_uint4(first, 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(rowp + ((c0 ^ 1u) << 4)) = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
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
    if (elect_one()) {
      prefetch_tmap(&tm_a);
      prefetch_tmap(&tm_bp);
      if (n_lr) {
        prefetch_tmap(&tm_xl1);
        prefetch_tmap(&tm_l2t);
      }
      const uint32_t main_tx = kI4BM * 64 + kI4BN * 32 + kI4BM * 2 + kI4BN * 4;
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
            bulk_load(st + kI4SwOff, p.sw16 + static_cast<size_t>(g) * p.N_pad + n0, kI4BN * 4, &full[s]);
          } else {
            const int c = step - p.groups;
            mbar_arrive_expect_tx(&full[s], lr_tx);
            tma_load_2d(st + kI4AOff, &tm_xl1, &full[s], c * 64, m0);
            tma_load_2d(st + kI4BOff, &tm_l2t, &full[s], c * 64, n0);
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
      const uint32_t c_a = smem_u32(smem + kI4ConstOff), c_b = c_a + 4096u, c_bn = c_a + 8192u;
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
          // the buffer := 1.5 * 2^23 (one bf16 MMA of the constant tiles); the
          // group's int8 products accumulate onto that offset's bits, which are
          // then the fp32 value 1.5 * 2^23 + 16 P; one more bf16 MMA adds
          // -1.5 * 2^23 in fp32 (exact), leaving the fp32 value 16 P
          mma_bf16(d, make_kmajor_desc(c_a, 32), make_kmajor_desc(c_b, 32), idesc_lr, 0u);
#pragma unroll
          for (int j = 0; j < 2; ++j)
            mma_i8(d, make_kmajor_desc(a0 + 32 * j, 64), make_kmajor_desc(b0 + 32 * j, 64), idesc_main, 1u);
          mma_bf16(d, make_kmajor_desc(c_a, 32), make_kmajor_desc(c_bn, 32), idesc_lr, 1u);
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
  } else if (warp >= 2 + kI4EpiWarps) {
    // ------------------------------------------------------------ unpack
    // Two warps (64 lanes) turn each landed stage's packed B (128 columns x 32
    // bytes) into the MMA layout: 64-byte rows, 64-byte swizzle (16-byte chunk
    // c of row r at c ^ ((r >> 1) & 3)).  Lane task t: 16 packed bytes (32
    // codes) = half h of row r -> unpacked chunks 2 h and 2 h + 1.
    const uint32_t ul = (warp - 2 - kI4EpiWarps) * 32 + lane;   // 0 .. 63
    bool ok = true;
    for (int u = 0; u < total_steps; ++u) {
      const int s = u % S;
      if (ok && !warp_wait(&full[s], (u / S) & 1, p.budget, abort_flag)) {
        if (lane == 0) raise_error(kErrWaitGemm);
        *abort_flag = 1;
        ok = false;
      }
      if (ok && (u % steps_per_tile) < p.groups) {
        uint8_t* st = smem + s * kI4StageBytes;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t t = ul + 64u * i;           // 0 .. 255
          const uint32_t r = t >> 1, hh = t & 1u;
          const uint4 w = *reinterpret_cast<const uint4*>(st + kI4BpOff + r * 32 + hh * 16);
          const uint2 a = i4_unpack8(w.x), b = i4_unpack8(w.y), c = i4_unpack8(w.z), d = i4_unpack8(w.w);
          const uint32_t sw = (r >> 1) & 3u;
          uint8_t* row = st + kI4BOff + r * 64;
          *reinterpret_cast<uint4*>(row + (((2 * hh) ^ sw) << 4)) = make_uint4(a.x, a.y, b.x, b.y);
          *reinterpret_cast<uint4*>(row + (((2 * hh + 1) ^ sw) << 4)) = make_uint4(c.x, c.y, d.x, d.y);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&unpacked[s]);
    }
  } else {
    // ------------------------------------------------------------ drain / epilogue
    const uint32_t q = warp & 3u;              // TMEM lane quarter this warp may access
    const uint32_t h = (warp - 2) >> 2;        // 64-column half of the tile
    const uint32_t row = q * 32 + lane;
    bool ok = true;
    int it = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
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
        if (ok && !warp_wait(&pfull[b], pph, p.budget, abort_flag)) {
          if (lane == 0) raise_error(kErrWaitGemm);
          *abort_flag = 1;
          ok = false;
        }
        if (ok) {
          tc_fence_after();
          const uint8_t* st = smem + s * kI4StageBytes;
          const uint32_t taddr = tmem_base + ((q * 32u) << 16) + kI4BN * b + 64u * h;
          const bool main_step = step < p.groups;
          unsigned long long sx2 = 0ull;
          if (main_step) {
            const float sx = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(st + kI4SxOff)[row]));
            sx2 = f2_pack(sx, sx);
          }
          const ulonglong2* sw4 = reinterpret_cast<const ulonglong2*>(st + kI4SwOff) + 16 * h;
          uint32_t r[64];
          tmem_ld64(taddr, r);   // one TMEM round trip per group
          tmem_wait_ld();
          if (main_step) {
            // acc += 16 P * (s_x * s_w / 16): the scale product and one fused
            // multiply-add per column pair; s_w / 16 read four columns at a time
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const ulonglong2 w4 = sw4[j / 2];   // s_w / 16 of columns 64 h + 2 j .. + 3
              acc[j] = f2_fma(u2_pack(r[2 * j], r[2 * j + 1]), f2_mul(sx2, w4.x), acc[j]);
              acc[j + 1] = f2_fma(u2_pack(r[2 * j + 2], r[2 * j + 3]), f2_mul(sx2, w4.y), acc[j + 1]);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[j] = f2_add(acc[j], u2_pack(r[2 * j], r[2 * j + 1]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&pempty[b]);
          mbar_arrive(&empty[s]);    // done with this stage's scales
        }
      }
      if (!ok) continue;   // keep walking the steps so the barriers stay matched
      // bias, bf16, store: 64 columns of this row
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
    mbar_wait(mma_done, 0, drain_budget(p.budget), nullptr);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace svdq
