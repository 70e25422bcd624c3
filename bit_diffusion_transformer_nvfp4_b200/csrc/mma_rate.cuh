// mma_rate.cuh -- the measured FP4 tensor-pipe rate: back-to-back block-scaled
// FP4 MMAs (tcgen05.mma kind::mxf4nvf4.block_scale.block16) on every SM with
// operands resident in shared memory and TMEM, no feed.  It gives the
// measured denominator of the FP4 roofline beside the nominal one (the
// measured bf16 rate times four).
//
// Pair mode: one cluster of two CTAs per two SMs, the even CTA issues
// 256 x 256 x 64 pair MMAs (cta_group::2) reading both CTAs' 128-row A tiles
// and 128-row halves of B.  Single mode: one CTA per SM, 128 x 256 x 64.
// Operands: pseudo-random code bytes (every byte is a pair of valid E2M1
// codes) and scale bytes between 0x30 and 0x3F (E4M3 0.5 .. 0.94), written
// before the timed loop; the MMAs cycle through the tile's four 64-deep K
// steps into one accumulator.  The issuing thread times its loop with the
// SM clock and waits (bounded) for the last MMA to complete.
#pragma once

#include "sm100.cuh"

namespace w4a4 {

constexpr int kRateThreads = 128;
constexpr int kRateABytes = 128 * 128;                   // 128 rows x 256 E2M1 codes
constexpr int kRateBBytes = 256 * 128;                   // 256 rows (single mode; a pair uses 128 per CTA)
constexpr int kRateSmem = kRateABytes + kRateBBytes + 256;  // A, B, barrier (1024-aligned base)
constexpr int kRateTmemCols = 512;                       // accumulator [0, 256), scales [256, 304)

__device__ __forceinline__ uint32_t rate_hash(uint32_t x) {
  x ^= x >> 16;
  x *= 0x7feb352dU;
  x ^= x >> 15;
  x *= 0x846ca68bU;
  x ^= x >> 16;
  return x;
}

template <bool PAIR>
__global__ void __launch_bounds__(kRateThreads, 1) fp4_mma_rate_kernel(int iters, unsigned long long* cycles,
                                                                      int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {  // the 128-byte swizzle needs 1024-byte aligned tiles
    if (threadIdx.x == 0) atomicExch(status, kStatusMisaligned);
    return;
  }
  uint8_t* sa = smem_raw;
  uint8_t* sb = smem_raw + kRateABytes;
  uint64_t* done = reinterpret_cast<uint64_t*>(smem_raw + kRateABytes + kRateBBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;

  // operands: pseudo-random code bytes
  const uint32_t seed = blockIdx.x * 0x9E3779B9u;
  for (int i = tid; i < (kRateABytes + kRateBBytes) / 4; i += kRateThreads)
    reinterpret_cast<uint32_t*>(sa)[i] = rate_hash(seed + static_cast<uint32_t>(i));
  fence_proxy_async_smem();
  if (tid == 0) {
    mbar_init(smem_u32(done), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(smem_u32(tmem_slot), kRateTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), kRateTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // scale bytes 0x30..0x3F in the 48 scale columns of every lane (A scales
  // at 4k, B scales at 16 + 8k for the K step k, as in the GEMM's slots)
  {
    uint32_t w[16];
#pragma unroll
    for (int h = 0; h < 3; ++h) {
#pragma unroll
      for (int c = 0; c < 16; ++c) w[c] = (rate_hash(seed ^ (tid * 64 + h * 16 + c)) & 0x0F0F0F0Fu) | 0x30303030u;
      tmem_st_16cols(tmem + (static_cast<uint32_t>(warp * 32) << 16) + 256 + 16 * h, w);
    }
    tmem_st_wait();
  }
  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();

  if (tid == 0 && rank == 0) {
    const uint32_t a0 = smem_u32(sa), b0 = smem_u32(sb);
    const uint32_t sf = tmem + 256;
    const uint32_t idesc = idesc_nvf4(PAIR ? 256 : 128, 256);
    const long long t0 = clock64();
    for (int it = 0; it < iters; ++it) {
      const int k = it & 3;
      const uint64_t ad = smem_desc(a0 + 32 * k, 16, 1024, kSwizzle128B);
      const uint64_t bd = smem_desc(b0 + 32 * k, 16, 1024, kSwizzle128B);
      if constexpr (PAIR)
        mma_nvf4_pair(tmem, ad, bd, idesc, sf + 4 * k, sf + 16 + 8 * k, it > 0 ? 1u : 0u);
      else
        mma_nvf4(tmem, ad, bd, idesc, sf + 4 * k, sf + 16 + 8 * k, it > 0 ? 1u : 0u);
    }
    if constexpr (PAIR) tc_commit_pair(smem_u32(done)); else tc_commit(smem_u32(done));
    const bool ok = mbar_wait(smem_u32(done), 0, abort_flag, status);
    const long long t1 = clock64();
    cycles[PAIR ? blockIdx.x / 2 : blockIdx.x] = ok ? static_cast<unsigned long long>(t1 - t0) : 0ull;
  }
  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem, kRateTmemCols); else tmem_dealloc(tmem, kRateTmemCols);
  }
}

}  // namespace w4a4
