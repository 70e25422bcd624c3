// gemm.cuh -- block-scaled FP4 GEMM with the low-rank branch, bias, optional
// GELU and the bf16 cast fused, on the sm_100a tensor cores.
//
// Structure (one persistent CTA per SM, 320 threads):
//   warp 0      TMA producer.  For every output tile (128 x BN) it first loads
//               the low-rank operands (U hi|lo [128 x 64] bf16, 128-byte
//               swizzle, and L2t [BN x 32] bf16, 64-byte swizzle) into one ring
//               stage, then for every 256-wide K step the FP4 codes of X and W
//               (128-byte rows, 128-byte swizzle) and their scale atoms
//               (2 KB + 4 KB, already in tensor-core order) into the next stage.
//   warp 1      TMEM allocator and MMA issuer (one elected lane).  Per tile:
//               four kind::f16 MMAs (K=16 each: hi part, then lo part against
//               the same L2t tile) initialise the fp32 accumulator with
//               U' L2; then per K step it copies the scale atoms into TMEM
//               (tcgen05.cp 32x128b.warpx4) and issues four
//               kind::mxf4nvf4.block16 MMAs (K=64 each) that accumulate
//               sum_k dec(Xq) dec(Xsf) dec(Wq) dec(Wsf) on top.  tcgen05.commit
//               frees each ring stage and finally hands the accumulator to
//               the epilogue.
//   warps 2-9   epilogue.  Warp w reads TMEM lanes 32*(w%4).. (its rows) and
//               half of the tile's columns, releases the accumulator as soon
//               as the values are in registers, then writes
//               bf16(t_x t_w acc + bias) (optionally through GELU) with 16-byte
//               stores.
// With BN = 192 the accumulator is double-buffered in TMEM (2 x 192 columns
// plus 48 scale columns), so the epilogue of one tile overlaps the main loop
// of the next; with BN = 256 it is single-buffered and the drain into
// registers is what the MMA warp waits for.
//
// The low-rank pass is the fused 4-bit + low-rank kernel idea of
// "SVDQuant Guide: 4-Bit DiT Acceleration & Outlier Absorption" (pillar 3,
// "The Nunchaku Fused Kernel Engine"), here done by accumulating both
// branches into one TMEM accumulator.
#pragma once

#include "sm100.cuh"

namespace w4a4 {

struct GemmParams {
  int M, N, K;
  int64_t ldy;
  const float* t_x;
  const float* t_w;
  const __nv_bfloat16* bias;
  __nv_bfloat16* Y;
  int has_lr;
  int r;  // low-rank rank: 0, 16 or 32
  int epi;
  int* status;
  // optional: the next layer's tensor amax max |fl(y * next_inv_s)| over the
  // stored bf16 outputs, atomically max-ed into *next_amax (as float bits;
  // non-negative floats order like their bit patterns).  next_inv_s may be
  // null (all ones).
  const float* next_inv_s;
  unsigned* next_amax;
  // SwiGLU epilogue (CTA-pair kernel only): weight rows [0, n_plain) give
  // plain outputs in Y; rows [n_plain, N) hold gate/up pairs in blocks of 32
  // (16 gate rows, then the 16 up rows of the same features), and the
  // kernel writes silu(gate) * up of each pair to H [M, (N - n_plain) / 2]
  // (row stride ldh).  n_plain == N: no SwiGLU columns.  With next_amax the
  // amax covers H only.
  int n_plain;
  __nv_bfloat16* H;
  int64_t ldh;
  // Quantise-into-epilogue (CTA-pair kernel only): the final outputs (Y, or
  // H in SwiGLU mode) are also written as the next layer's NVFP4 codes and
  // block scales under the given tensor scale *t_next, smoothed by
  // next_inv_s: output column c is column q_col0 + c of the next layer's
  // [M, next_K] activation (codes q_next [M, ldq bytes], SF atoms sf_next).
  // q_next == nullptr: off.  Y / H == nullptr: the bf16 values are not stored.
  uint8_t* q_next;
  uint8_t* sf_next;
  const float* t_next;
  int64_t ldq;
  int next_K;
  int q_col0;
  // Rotary embedding (CTA-pair kernel, ROPE instantiation): plain outputs
  // n < n_rope form heads of d_head features; features 2i, 2i+1 of a head
  // are turned by the angle whose (cos, sin) are rope[m * ld_rope + 2i],
  // rope[m * ld_rope + 2i + 1] for token m.  n_rope == 0: off.
  int n_rope;
  int d_head;
  const float* rope;
  int64_t ld_rope;
};

// Shared-memory descriptors of the low-rank pass, K step k (16 columns) of
// U = [hi | lo] (rows of 2r bf16: 128-byte swizzle at rank 32, 64-byte at
// rank 16) against L2t (rows of r bf16: 64-byte / 32-byte swizzle), whose
// columns are used once for the hi and once for the lo half.
__device__ __forceinline__ uint64_t lowrank_desc_u(uint32_t base, int k, int r) {
  return r == 32 ? smem_desc(base + 32 * k, 16, 1024, kSwizzle128B) : smem_desc(base + 32 * k, 16, 512, kSwizzle64B);
}
__device__ __forceinline__ uint64_t lowrank_desc_l2(uint32_t base, int k, int r) {
  return r == 32 ? smem_desc(base + 32 * (k & 1), 16, 512, kSwizzle64B) : smem_desc(base, 16, 256, kSwizzle32B);
}

// Fold eight stored bf16 outputs (columns n .. n+7) into a running amax of
// |y * s| (s > 0, so |fl(y s)| = fl(|y| s)).
__device__ __forceinline__ float amax_fold8(float m, uint4 o, const float* next_inv_s, int n) {
  const uint32_t w[4] = {o.x, o.y, o.z, o.w};
  float v[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    v[2 * j] = fabsf(bf16_lo(w[j]));
    v[2 * j + 1] = fabsf(bf16_hi(w[j]));
  }
  if (next_inv_s != nullptr) {
    const float4 s0 = __ldg(reinterpret_cast<const float4*>(next_inv_s + n));
    const float4 s1 = __ldg(reinterpret_cast<const float4*>(next_inv_s + n + 4));
    v[0] = __fmul_rn(v[0], s0.x); v[1] = __fmul_rn(v[1], s0.y); v[2] = __fmul_rn(v[2], s0.z);
    v[3] = __fmul_rn(v[3], s0.w); v[4] = __fmul_rn(v[4], s1.x); v[5] = __fmul_rn(v[5], s1.y);
    v[6] = __fmul_rn(v[6], s1.z); v[7] = __fmul_rn(v[7], s1.w);
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) m = fmaxf(m, v[j]);
  return m;
}

// One atomic max per warp of the lanes' running maxima.
__device__ __forceinline__ void amax_publish(float m, unsigned* next_amax) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0 && next_amax != nullptr) atomicMax(next_amax, __float_as_uint(m));
}

template <int BN_, int STAGES_>
struct GemmCfg {
  static constexpr int BN = BN_;
  static constexpr int STAGES = STAGES_;
  static constexpr int BM = 128;
  static constexpr int BK = 256;                       // FP4 elements per ring stage
  static constexpr int A_BYTES = BM * 128;             // 128 rows x 128 bytes
  static constexpr int B_BYTES = BN * 128;
  static constexpr int SFA_BYTES = 4 * 512;            // 4 atoms (one per K=64)
  static constexpr int SFB_BYTES = 2 * 4 * 512;        // 2 row blocks x 4 atoms
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int LR_BYTES = BM * 128 + BN * 64;  // U tile + L2t tile at rank 32 (rank 16: half)
  static constexpr int NUM_ACC = (2 * BN + 48 <= 512) ? 2 : 1;
  static constexpr int SFA_COL = NUM_ACC * BN;
  static constexpr int SFB_COL = SFA_COL + 16;
  static constexpr int TMEM_COLS = 512;
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int HALF = BN / 2;                  // columns per epilogue warp
  static constexpr int SMEM = STAGE_BYTES * STAGES + 1024 + 256;
  static_assert(SFB_COL + 32 <= TMEM_COLS, "TMEM budget");
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
  static_assert(HALF % 32 == 0, "epilogue column split");
};

// GELU, tanh form: 0.5 y (1 + tanh(u)), u = sqrt(2/pi) (y + 0.044715 y^3).
// With t = exp(-2|u|) in (0, 1] the same value is y / (1 + t) for y >= 0 and
// y t / (1 + t) for y < 0: no cancellation on either side (1 + tanh(u) for
// large negative y would lose all its digits), no overflow (t underflows to 0
// for large |y|, giving y and -0), and no IEEE division (its slow path made
// the epilogue the bottleneck).  The hardware base-2 exponential and
// reciprocal keep the result within a few fp32 ulps, far inside the bf16
// rounding of the output.
__device__ __forceinline__ float gelu_tanh_f32(float y) {
  const float u = 0.7978845608028654f * (y + 0.044715f * y * y * y);
  const float t = ex2_approx(-2.8853900817779268f * fabsf(u));  // exp(-2|u|) = 2^(-2 log2(e) |u|)
  const float num = y < 0.0f ? y * t : y;
  return num * rcp_approx(1.0f + t);
}

// silu(y) = y sigmoid(y).  With t = exp(-|y|) in (0, 1] it equals y / (1 + t)
// for y >= 0 and y t / (1 + t) for y < 0: no overflow (t underflows to 0 for
// large |y|, giving y and -0) and no IEEE division; the hardware base-2
// exponential and reciprocal keep it within a few fp32 ulps.
__device__ __forceinline__ float silu_f32(float y) {
  const float t = ex2_approx(-1.4426950408889634f * fabsf(y));  // exp(-|y|) = 2^(-log2(e) |y|)
  const float num = y < 0.0f ? y * t : y;
  return num * rcp_approx(1.0f + t);
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
                const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_l2,
                const GemmParams p) {
  constexpr int BN = C::BN, STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGE_BYTES * STAGES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + C::NUM_ACC;
  uint64_t* drain = acc_empty + C::NUM_ACC;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool lr = p.has_lr != 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < C::NUM_ACC; ++a) {
      mbar_init(smem_u32(&acc_full[a]), 1);
      mbar_init(smem_u32(&acc_empty[a]), C::EPI_WARPS);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_sfa);
    tma_prefetch_desc(&tm_sfb);
    if (lr) {
      tma_prefetch_desc(&tm_u);
      tma_prefetch_desc(&tm_l2);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // set-up above overlaps the tail of the previous kernel in the stream
  // (programmatic launch); nothing below may touch memory before this
  grid_dependency_wait();

  const int m_tiles = (p.M + C::BM - 1) / C::BM;
  const int n_tiles = (p.N + BN - 1) / BN;
  const int total = m_tiles * n_tiles;
  const int nkb = (p.K + C::BK - 1) / C::BK;  // the last K step may be partial: TMA fills zeros

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const int m0 = (tile % m_tiles) * C::BM;
        const int n0 = (tile / m_tiles) * BN;
        if (lr) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, abort_flag, p.status)) { ok = false; break; }
          uint8_t* st = smem + s * C::STAGE_BYTES;
          const uint32_t bar = smem_u32(&full[s]);
          mbar_arrive_expect_tx(bar, C::LR_BYTES * p.r / 32);
          tma_load_2d(smem_u32(st), &tm_u, bar, 0, m0);
          tma_load_2d(smem_u32(st + C::A_BYTES), &tm_l2, bar, 0, n0);
          ++it;
        }
        for (int kb = 0; kb < nkb; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, abort_flag, p.status)) { ok = false; break; }
          uint8_t* st = smem + s * C::STAGE_BYTES;
          const uint32_t bar = smem_u32(&full[s]);
          mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
          tma_load_2d(smem_u32(st), &tm_a, bar, kb * 128, m0);
          tma_load_2d(smem_u32(st + C::A_BYTES), &tm_b, bar, kb * 128, n0);
          tma_load_3d(smem_u32(st + C::A_BYTES + C::B_BYTES), &tm_sfa, bar, 0, kb * 4, m0 / 128);
          tma_load_3d(smem_u32(st + C::A_BYTES + C::B_BYTES + C::SFA_BYTES), &tm_sfb, bar, 0, kb * 4,
                      n0 / 128);
          ++it;
        }
      }
      // Fills still in flight (only possible after an abort) must land before
      // the shared memory is released.
      const uint32_t first = it > static_cast<uint32_t>(STAGES) ? it - STAGES : 0u;
      for (uint32_t j = first; j < it; ++j) mbar_wait_drain(smem_u32(&full[j % STAGES]), (j / STAGES) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescF4 = idesc_nvf4(128, BN);
      constexpr uint32_t kIdescBf = idesc_bf16(128, BN);
      uint32_t it = 0, tcount = 0;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        const int n0 = (tile / m_tiles) * BN;
        const uint32_t acc = tcount % C::NUM_ACC;
        const uint32_t aph = (tcount / C::NUM_ACC) & 1;
        if (!mbar_wait(smem_u32(&acc_empty[acc]), aph ^ 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        const uint32_t sfb_shift = static_cast<uint32_t>((n0 % 128) / 32);
        bool first = true;
        bool ok = true;
        if (lr) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(smem_u32(&full[s]), ph, abort_flag, p.status)) break;
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + s * C::STAGE_BYTES);
          const uint32_t b_base = a_base + C::A_BYTES;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            if (k < p.r / 8) mma_bf16(d, lowrank_desc_u(a_base, k, p.r), lowrank_desc_l2(b_base, k, p.r), kIdescBf, k > 0 ? 1u : 0u);
          }
          tc_commit(smem_u32(&empty[s]));
          ++it;
          first = false;
        }
        for (int kb = 0; kb < nkb; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(smem_u32(&full[s]), ph, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + s * C::STAGE_BYTES);
          const uint32_t b_base = a_base + C::A_BYTES;
          const uint32_t sfa_base = b_base + C::B_BYTES;
          const uint32_t sfb_base = sfa_base + C::SFA_BYTES;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tc_cp_32x128b_x4(tmem + C::SFA_COL + 4 * j, smem_desc(sfa_base + 512 * j, 0, 128, kSwizzleNone));
            tc_cp_32x128b_x4(tmem + C::SFB_COL + 8 * j, smem_desc(sfb_base + 512 * j, 0, 128, kSwizzleNone));
            tc_cp_32x128b_x4(tmem + C::SFB_COL + 8 * j + 4,
                             smem_desc(sfb_base + 2048 + 512 * j, 0, 128, kSwizzleNone));
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t ad = smem_desc(a_base + 32 * j, 16, 1024, kSwizzle128B);
            const uint64_t bd = smem_desc(b_base + 32 * j, 16, 1024, kSwizzle128B);
            mma_nvf4(d, ad, bd, kIdescF4, tmem + C::SFA_COL + 4 * j, tmem + C::SFB_COL + 8 * j + sfb_shift,
                     (!first || j > 0) ? 1u : 0u);
          }
          tc_commit(smem_u32(&empty[s]));
          ++it;
          first = false;
        }
        if (!ok) break;
        tc_commit(smem_u32(&acc_full[acc]));
        ++tcount;
      }
      // Every MMA issued by this thread completes before TMEM is released.
      tc_commit(smem_u32(drain));
      mbar_wait_drain(smem_u32(drain), 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;               // TMEM lane quarter this warp may access
    const int h = (warp - 2) >> 2;        // column half
    const float alpha = __fmul_rn(__ldg(p.t_x), __ldg(p.t_w));
    float amax = 0.0f;  // next layer's amax over this thread's stored outputs
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const int m0 = (tile % m_tiles) * C::BM;
      const int n0 = (tile / m_tiles) * BN;
      const uint32_t acc = tcount % C::NUM_ACC;
      const uint32_t aph = (tcount / C::NUM_ACC) & 1;
      if (!mbar_wait(smem_u32(&acc_full[acc]), aph, abort_flag, p.status)) break;
      tc_fence_after();
      uint32_t r[C::HALF];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + h * C::HALF;
#pragma unroll
      for (int c = 0; c < C::HALF / 32; ++c)
        tmem_ld_32cols(taddr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acc_empty[acc]));

      const int row = m0 + q * 32 + lane;
      if (row < p.M) {
        __nv_bfloat16* yrow = p.Y + static_cast<int64_t>(row) * p.ldy;
#pragma unroll
        for (int g = 0; g < C::HALF / 8; ++g) {
          const int n = n0 + h * C::HALF + 8 * g;
          if (n < p.N) {
            float b[8];
            if (p.bias != nullptr) {
              const uint4 bw = __ldg(reinterpret_cast<const uint4*>(p.bias + n));
              b[0] = bf16_lo(bw.x); b[1] = bf16_hi(bw.x); b[2] = bf16_lo(bw.y); b[3] = bf16_hi(bw.y);
              b[4] = bf16_lo(bw.z); b[5] = bf16_hi(bw.z); b[6] = bf16_lo(bw.w); b[7] = bf16_hi(bw.w);
            } else {
#pragma unroll
              for (int j = 0; j < 8; ++j) b[j] = 0.0f;
            }
            float y[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              y[j] = __fadd_rn(__fmul_rn(alpha, __uint_as_float(r[8 * g + j])), b[j]);
              if (p.epi == 1) y[j] = gelu_tanh_f32(y[j]);
            }
            uint4 o;
            o.x = pack_bf16x2(y[0], y[1]);
            o.y = pack_bf16x2(y[2], y[3]);
            o.z = pack_bf16x2(y[4], y[5]);
            o.w = pack_bf16x2(y[6], y[7]);
            *reinterpret_cast<uint4*>(yrow + n) = o;
            if (p.next_amax != nullptr) amax = amax_fold8(amax, o, p.next_inv_s, n);
          }
        }
      }
      ++tcount;
    }
    if (p.next_amax != nullptr) amax_publish(amax, p.next_amax);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace w4a4
