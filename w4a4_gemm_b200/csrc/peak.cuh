// peak.cuh -- the tensor-core ceiling the GEMM rooflines are read against.
//
// Every SM issues the GEMM's own MMA shape back to back from operands already
// in shared memory (no global loads, no epilogue), so the rate a caller times
// around this kernel is what the tensor cores sustain on this part, under its
// power cap, for that instruction:
//   NVFP4: tcgen05.mma kind::mxf4nvf4 block16, M=128 N=256 K=64 (4 per 256-wide K step)
//   INT4 : tcgen05.mma kind::i8,                 M=128 N=256 K=32
// The operands hold a fixed pseudo-random pattern (all-zero data would draw
// less power than real codes).
#pragma once

#include "svdq_formats.cuh"
#include "svdq_ptx.cuh"

namespace svdq {

constexpr int kPeakThreads = 128;
constexpr uint32_t kPeakAOff = 0;            // 128 rows x 128 B
constexpr uint32_t kPeakBOff = 16384;        // 256 rows x 128 B
constexpr uint32_t kPeakSfOff = 49152;       // 12 scale atoms of 512 B
constexpr uint32_t kPeakSmemBytes = 49152 + 12 * 512 + 64 + 1024;

template <int FMT>
__global__ void __launch_bounds__(kPeakThreads, 1)
    tensor_peak_kernel(long long n_steps, long long budget) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint64_t* done = reinterpret_cast<uint64_t*>(smem + kPeakSfOff + 12 * 512);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);
  const uint32_t warp = warp_id();

  for (uint32_t i = threadIdx.x; i < kPeakSfOff; i += kPeakThreads) {
    uint32_t h = (i + 0x9E3779B9u * (blockIdx.x + 1)) * 0x85EBCA6Bu;
    h ^= h >> 13;
    // NVFP4: any byte is two valid E2M1 codes; INT4: int8 codes in [-7, 7]
    smem[i] = FMT == 0 ? static_cast<uint8_t>(h) : static_cast<uint8_t>(static_cast<int>(h % 15u) - 7);
  }
  for (uint32_t i = threadIdx.x; i < 12 * 512; i += kPeakThreads)
    smem[kPeakSfOff + i] = static_cast<uint8_t>(0x30 + (i * 7) % 16);   // E4M3 0.5 .. 1.875
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0 && elect_one()) {
    const uint32_t a0 = smem_u32(smem + kPeakAOff), b0 = smem_u32(smem + kPeakBOff);
    if (FMT == 0) {
      const uint32_t sf = smem_u32(smem + kPeakSfOff);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        tmem_cp_32x128b_x4(tmem_base + 256 + 4 * j, make_sdesc(sf + 512 * j, 0, 128, kSwizzleNone));
        tmem_cp_32x128b_x4(tmem_base + 272 + 8 * j, make_sdesc(sf + 2048 + 512 * j, 0, 128, kSwizzleNone));
        tmem_cp_32x128b_x4(tmem_base + 276 + 8 * j, make_sdesc(sf + 4096 + 512 * j, 0, 128, kSwizzleNone));
      }
      const uint32_t idesc = idesc_e2m1_ue4m3(128, 256);
      for (long long s = 0; s < n_steps; ++s) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_nvf4(tmem_base, make_kmajor_desc(a0 + 32 * j, 128), make_kmajor_desc(b0 + 32 * j, 128),
                   idesc, tmem_base + 256 + 4 * j, tmem_base + 272 + 8 * j, (s > 0 || j > 0) ? 1u : 0u);
      }
    } else {
      const uint32_t idesc = idesc_s8_s32(128, 256);
      for (long long s = 0; s < n_steps; ++s) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_i8(tmem_base, make_kmajor_desc(a0 + 32 * j, 128), make_kmajor_desc(b0 + 32 * j, 128),
                 idesc, (s > 0 || j > 0) ? 1u : 0u);
      }
    }
    tc_commit(done);
  }
  __syncwarp();
  if (warp == 0) {
    // the MMAs run for the whole measurement: wait for them before freeing TMEM
    if (!warp_wait(done, 0, drain_budget(budget), nullptr) && lane_id() == 0) raise_error(kErrWaitOther);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace svdq
