// attention.cuh -- FP8 attention on the sm_100a tensor cores, and the FP8
// tensor quantiser that feeds it.
//
// The NVIDIA blog page on FLUX on Blackwell quantises attention to FP8 after
// the NVFP4 GEMMs ("NVIDIA Technical Blog Details FLUX 3 Image Klein
// Blackwell Inference Optimization Methods": VC-Attention FP8), without the
// arithmetic.  Here: queries, keys and values in E4M3 with one fp32 scale per
// tensor; per (128-query tile, head, sequence) one CTA computes
//   S = Q K^T            tcgen05.mma kind::f8f6f4 (E4M3 x E4M3, fp32 in TMEM)
//   P = 2^(c S - m)      online softmax in fp32 (c = scale s_q s_k log2 e),
//                        rounded to E4M3 for the second product
//   O = sum_j P_j V_j    tcgen05.mma kind::f8f6f4 into a second TMEM accumulator
// and writes bf16 O s_v / l (l = the sum of P before the rounding).  The running
// offset m moves only when a tile's maximum exceeds it by more than half a
// binade, and sits 8 binades above the largest probability so that E4M3's
// range holds P from 2^-17 to 2^8.5 of the row's largest weight; O and l are
// rescaled in TMEM / registers when it moves.
//
// Roles (192 threads, two CTAs per SM): warp 0 TMA producer (the query tile
// once, then key and value tiles through a two-stage ring), warp 1 TMEM owner
// and the single MMA-issuing thread, warps 2-5 softmax (one query row per
// thread: TMEM lane quarter warp % 4).  A softmax thread copies its row's 128
// scores into registers at once, so the next tile's Q K^T runs on the tensor
// cores while this tile's probabilities are computed.
#pragma once

#include "sm100.cuh"

namespace w4a4 {

constexpr int kAttnD = 128;          // head size
constexpr int kAttnTile = 128;       // queries per CTA, keys per step
constexpr int kAttnStages = 2;       // key/value stages
constexpr int kAttnThreads = 192;
constexpr int kAttnSoftmaxWarp0 = 2;
constexpr int kAttnTmemCols = 256;   // S [0, 128), O [128, 256)
constexpr float kAttnOffset = 8.0f;  // binades between the running maximum and P = 1
constexpr float kAttnSlack = 0.5f;   // a tile maximum this far above the offset's maximum moves it

struct AttnParams {
  int S;               // tokens per sequence (multiple of 128)
  int heads;
  const float* s_q;    // per-tensor dequantisation scales
  const float* s_k;
  const float* s_v;
  float scale;         // softmax scale (1/sqrt(d))
  __nv_bfloat16* O;    // [B * S, ldo], head h in columns h*128 ..
  int64_t ldo;
  int* status;
};

struct AttnSmem {
  static constexpr int kTileBytes = kAttnTile * kAttnD;     // 16 KB of E4M3
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kTileBytes;                  // stages: K, then V^T
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kPOff = kKOff + kAttnStages * kStageBytes;
  static constexpr int kBarOff = kPOff + kTileBytes;
  static constexpr int kBytes = kBarOff + 256 + 1024;
  static_assert(kBytes <= 113 * 1024, "two CTAs per SM");
};

// FP8 instruction descriptor: fp32 accumulate, E4M3 A and B, K-major.
constexpr uint32_t idesc_e4m3(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_e4m3(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Blackwell packed fp32 fused multiply-add and add: two IEEE round-to-nearest results.
__device__ __forceinline__ void fma2_rn(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                        float c1) {
  asm("{\n\t.reg .b64 a, b, c, d;\n\t"
      "mov.b64 a, {%2, %3};\n\t"
      "mov.b64 b, {%4, %5};\n\t"
      "mov.b64 c, {%6, %7};\n\t"
      "fma.rn.f32x2 d, a, b, c;\n\t"
      "mov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void add2_rn(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\t"
      "mov.b64 a, {%2, %3};\n\t"
      "mov.b64 b, {%4, %5};\n\t"
      "add.rn.f32x2 d, a, b;\n\t"
      "mov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// 2^x for two values on the FMA and integer pipes instead of the MUFU:
// n = round(x) from the sum with 1.5 * 2^23, f = x - n in [-1/2, 1/2], a cubic
// in f (fitted to 2^f on [-1/2, 1/2] by iteratively reweighted least squares
// on the relative error: at most 7.5e-5, far below the E4M3 rounding that
// follows) scaled by 2^n through the exponent field.  x is clamped at -126,
// where the result is far below the smallest E4M3 value anyway.
__device__ __forceinline__ void exp2_poly2(float& y0, float& y1, float x0, float x1) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  constexpr float c0 = 0.99992758f, c1 = 0.69326109f, c2 = 0.24261758f, c3 = 0.05517415f;
  x0 = fmaxf(x0, -126.0f);
  x1 = fmaxf(x1, -126.0f);
  float t0, t1, n0, n1, f0, f1, p0, p1;
  add2_rn(t0, t1, x0, x1, kMagic, kMagic);
  add2_rn(n0, n1, t0, t1, -kMagic, -kMagic);
  add2_rn(f0, f1, x0, x1, -n0, -n1);
  fma2_rn(p0, p1, f0, f1, c3, c3, c2, c2);
  fma2_rn(p0, p1, p0, p1, f0, f1, c1, c1);
  fma2_rn(p0, p1, p0, p1, f0, f1, c0, c0);
  const int kb = __float_as_int(kMagic);
  y0 = __int_as_float(__float_as_int(p0) + ((__float_as_int(t0) - kb) << 23));
  y1 = __int_as_float(__float_as_int(p1) + ((__float_as_int(t1) - kb) << 23));
}

// Each thread of the warp reads 16 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_ld_16cols(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Each thread of the warp writes 32 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_st_32cols(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// grid (S / 128 query tiles, heads, sequences).  Q and K: E4M3 [B*S, H*128]
// token-major (box 128 x 128); V^T: E4M3 [H*128, B*S] (box 128 keys x 128
// features); all 128-byte swizzled.
__global__ void __launch_bounds__(kAttnThreads, 2) attn_fp8_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                                 const __grid_constant__ CUtensorMap tm_k,
                                                                 const __grid_constant__ CUtensorMap tm_vt,
                                                                 const AttnParams p) {
  using L = AttnSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* q_full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* kv_full = q_full + 1;               // [stages]
  uint64_t* kv_free = kv_full + kAttnStages;    // [stages] the tile's MMAs are done
  uint64_t* s_full = kv_free + kAttnStages;     // S of the current tile is in TMEM
  uint64_t* s_free = s_full + 1;                // the softmax warps have read S
  uint64_t* p_full = s_free + 1;                // P is in shared memory, O rescaled
  uint64_t* o_done = p_full + 1;                // the P V MMAs of the tile are done
  uint64_t* drain = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q_tile = blockIdx.x, head = blockIdx.y, seq = blockIdx.z;
  const int n_kv = p.S / kAttnTile;
  const int row0 = seq * p.S + q_tile * kAttnTile;  // first query row
  const int key0 = seq * p.S;

  if (tid == 0) {
    mbar_init(smem_u32(q_full), 1);
    for (int s = 0; s < kAttnStages; ++s) {
      mbar_init(smem_u32(&kv_full[s]), 1);
      mbar_init(smem_u32(&kv_free[s]), 1);
    }
    mbar_init(smem_u32(s_full), 1);
    mbar_init(smem_u32(s_free), 4);
    mbar_init(smem_u32(p_full), 4);
    mbar_init(smem_u32(o_done), 1);
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kAttnTmemCols);
    tmem_relinquish();
  }
  grid_dependency_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_s = tmem, t_o = tmem + kAttnTile;

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_vt);
      mbar_arrive_expect_tx(smem_u32(q_full), L::kTileBytes);
      tma_load_2d(smem_u32(smem + L::kQOff), &tm_q, smem_u32(q_full), head * kAttnD, row0);
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % kAttnStages;
        if (j >= kAttnStages &&
            !mbar_wait(smem_u32(&kv_free[s]), ((j / kAttnStages) - 1) & 1, abort_flag, p.status))
          break;
        uint8_t* st = smem + L::kKOff + s * L::kStageBytes;
        const uint32_t bar = smem_u32(&kv_full[s]);
        mbar_arrive_expect_tx(bar, 2 * L::kTileBytes);
        tma_load_2d(smem_u32(st), &tm_k, bar, head * kAttnD, key0 + j * kAttnTile);
        tma_load_2d(smem_u32(st + L::kTileBytes), &tm_vt, bar, key0 + j * kAttnTile, head * kAttnD);
      }
      // every fill issued must land before the shared memory is released
      for (int j = max(0, n_kv - kAttnStages); j < n_kv; ++j)
        mbar_wait_drain(smem_u32(&kv_full[j % kAttnStages]), (j / kAttnStages) & 1);
      mbar_wait_drain(smem_u32(q_full), 0);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_e4m3(kAttnTile, kAttnTile);
      const uint32_t q_base = smem_u32(smem + L::kQOff), p_base = smem_u32(smem + L::kPOff);
      // S = Q K_j^T for tile j once its keys have landed and the softmax
      // warps hold tile j-1's scores in registers
      auto issue_s = [&](int j) -> bool {
        const int s = j % kAttnStages;
        if (!mbar_wait(smem_u32(&kv_full[s]), (j / kAttnStages) & 1, abort_flag, p.status) ||
            (j > 0 && !mbar_wait(smem_u32(s_free), (j - 1) & 1, abort_flag, p.status)))
          return false;
        tc_fence_after();
        const uint32_t k_base = smem_u32(smem + L::kKOff + s * L::kStageBytes);
#pragma unroll
        for (int k = 0; k < kAttnD / 32; ++k)
          mma_e4m3(t_s, smem_desc(q_base + 32 * k, 16, 1024, kSwizzle128B),
                   smem_desc(k_base + 32 * k, 16, 1024, kSwizzle128B), idesc, k > 0 ? 1u : 0u);
        tc_commit(smem_u32(s_full));
        return true;
      };
      bool ok = mbar_wait(smem_u32(q_full), 0, abort_flag, p.status) && (n_kv == 0 || issue_s(0));
      for (int j = 0; j < n_kv && ok; ++j) {
        const int s = j % kAttnStages;
        const uint32_t v_base = smem_u32(smem + L::kKOff + s * L::kStageBytes) + L::kTileBytes;
        // the next tile's scores overlap this tile's softmax
        if (j + 1 < n_kv && !issue_s(j + 1)) break;
        if (!mbar_wait(smem_u32(p_full), j & 1, abort_flag, p.status)) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < kAttnTile / 32; ++k)
          mma_e4m3(t_o, smem_desc(p_base + 32 * k, 16, 1024, kSwizzle128B),
                   smem_desc(v_base + 32 * k, 16, 1024, kSwizzle128B), idesc, (j > 0 || k > 0) ? 1u : 0u);
        tc_commit(smem_u32(o_done));
        tc_commit(smem_u32(&kv_free[s]));
      }
      tc_commit(smem_u32(drain));
      mbar_wait_drain(smem_u32(drain), 0);
    }
  } else {
    // ------------------------------------------------------- softmax, one query row per thread
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const float c = p.scale * __ldg(p.s_q) * __ldg(p.s_k) * 1.4426950408889634f;  // log2 e
    uint8_t* prow = smem + L::kPOff + (r >> 3) * 1024 + (r & 7) * 128;
    float m_used = -INFINITY;  // log2-domain offset base: P = 2^(c s - m_used + 8)
    float l = 0.0f;
    bool ok = true;
    // The tcgen05.ld / tcgen05.st below are warp-collective (.sync.aligned):
    // every branch around them is taken by the whole warp.
    for (int j = 0; j < n_kv; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(s_full), j & 1, abort_flag, p.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // the row's 128 scores into registers, and S's TMEM columns free for
      // the next tile's Q K^T while this one's softmax runs
      uint32_t sv[kAttnTile];
#pragma unroll
      for (int cc = 0; cc < kAttnTile / 32; ++cc)
        tmem_ld_32cols(t_s + lane_base + 32 * cc, *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * cc]));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(s_free));
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int i = 0; i < kAttnTile; ++i) mx4[i & 3] = fmaxf(mx4[i & 3], __uint_as_float(sv[i]));
      const float m_tile = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * c;
      // the previous tile's P V products must be done before P is rewritten
      // or O is read
      if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(smem_u32(o_done), (j - 1) & 1, abort_flag, p.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // rows whose tile maximum passed the offset's move it; O and l of
      // such a row scale by 2^(m_used - m_tile) (the first tile sets it)
      const bool moves = m_tile > m_used + kAttnSlack;
      const float m_new = moves ? m_tile : m_used;
      const float f = (j > 0 && moves) ? ex2_approx(m_used - m_new) : 1.0f;
      if (__any_sync(0xffffffffu, j > 0 && moves)) {
        l *= f;
        // 16 columns at a time: the row's scores stay in registers meanwhile
#pragma unroll 1
        for (int cc = 0; cc < kAttnD / 16; ++cc) {
          uint32_t v[16];
          tmem_ld_16cols(t_o + lane_base + 16 * cc, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * f);
          tmem_st_16cols(t_o + lane_base + 16 * cc, v);
        }
        tmem_st_wait();
      }
      m_used = m_new;
      const float off = m_used - kAttnOffset;
      // P = 2^(c s - off) in E4M3, 32 keys at a time, into the row of the
      // swizzled P tile; l sums the probabilities (the rounding to E4M3 is
      // unbiased, so the sum of the rounded ones differs from it far less
      // than each product does)
      float la = 0.0f, lb = 0.0f;
#pragma unroll
      for (int cc = 0; cc < kAttnTile / 32; ++cc) {
        uint32_t b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t* v = &sv[32 * cc + 4 * i];
          float x0, x1, x2, x3;
          fma2_rn(x0, x1, __uint_as_float(v[0]), __uint_as_float(v[1]), c, c, -off, -off);
          fma2_rn(x2, x3, __uint_as_float(v[2]), __uint_as_float(v[3]), c, c, -off, -off);
          // one pair in eight values on the FMA pipes, the rest on the MUFU
          float p0, p1;
          if ((i & 1) == 0) {
            exp2_poly2(p0, p1, x0, x1);
          } else {
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          const float p2 = ex2_approx(x2), p3 = ex2_approx(x3);
          b[i] = cvt_e4m3x2(p1, p0) | (cvt_e4m3x2(p3, p2) << 16);
          float s0, s1;
          add2_rn(s0, s1, p0, p1, p2, p3);
          add2_rn(la, lb, la, lb, s0, s1);
        }
        // keys 32cc .. 32cc+31: 16-byte units 2cc and 2cc+1 of the row
#pragma unroll
        for (int u = 0; u < 2; ++u)
          *reinterpret_cast<uint4*>(prow + (((2 * cc + u) ^ (r & 7)) << 4)) =
              make_uint4(b[4 * u], b[4 * u + 1], b[4 * u + 2], b[4 * u + 3]);
      }
      l += la + lb;
      fence_proxy_async_smem();  // P written by this thread, read by the tensor core
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(p_full));
    }
    if (ok && n_kv > 0 && __all_sync(0xffffffffu, mbar_wait(smem_u32(o_done), (n_kv - 1) & 1, abort_flag, p.status))) {
      tc_fence_after();
      // O / l, times the value scale, to bf16: 256 bytes of the row
      const float f = __ldg(p.s_v) / l;
      __nv_bfloat16* orow = p.O + static_cast<int64_t>(row0 + r) * p.ldo + head * kAttnD;
#pragma unroll 1
      for (int cc = 0; cc < kAttnD / 32; ++cc) {
        uint32_t v[32];
        tmem_ld_32cols(t_o + lane_base + 32 * cc, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(v[8 * i]) * f, __uint_as_float(v[8 * i + 1]) * f);
          w.y = pack_bf16x2(__uint_as_float(v[8 * i + 2]) * f, __uint_as_float(v[8 * i + 3]) * f);
          w.z = pack_bf16x2(__uint_as_float(v[8 * i + 4]) * f, __uint_as_float(v[8 * i + 5]) * f);
          w.w = pack_bf16x2(__uint_as_float(v[8 * i + 6]) * f, __uint_as_float(v[8 * i + 7]) * f);
          *reinterpret_cast<uint4*>(orow + 32 * cc + 8 * i) = w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kAttnTmemCols);
  }
}

// ------------------------------------------------------------------ FP8 tensor quantiser
// codes = E4M3_rn_satfinite(fl(x * fl(1 / s))), s = amax / 448 (1 when not a
// normal number), amax the maximum of the pass-1 partials.  Tiles of 128 rows
// x 64 columns; with `transpose` the codes of column c, row r go to
// out[c * ldo + r] (through shared memory, 128-byte row segments out).
struct Fp8QuantParams {
  const __nv_bfloat16* X;
  int64_t rows, cols, ldx;
  uint8_t* out;
  int64_t ldo;
  const float* partials;
  int n_partials;
  float* scale_out;
  int transpose;
};

__device__ __forceinline__ float fp8_scale_from(float amax) {
  float s = __fdiv_rn(amax, 448.0f);
  if (!(s >= 1.17549435e-38f)) s = 1.0f;
  return s;
}

__global__ void __launch_bounds__(256) fp8_quant_kernel(const Fp8QuantParams p) {
  __shared__ float red[8];
  __shared__ __align__(16) uint8_t tile[64][128 + 16];  // [column][row] when transposing
  const int tid = threadIdx.x, lane = tid & 31;
  float m = 0.0f;
  for (int i = tid; i < p.n_partials; i += 256) m = fmaxf(m, p.partials[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[tid >> 5] = m;
  __syncthreads();
  float amax = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
  const float s = fp8_scale_from(amax);
  const float inv = __frcp_rn(s);
  if (blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) *p.scale_out = s;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * 128, c0 = static_cast<int64_t>(blockIdx.x) * 64;
  // 128 rows x 64 columns: 8 threads of 8 columns per row, 32 rows per pass
  const int cseg = tid & 7, rsub = tid >> 3;
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    const int rr = pass * 32 + rsub;
    const int64_t row = r0 + rr, col = c0 + 8 * cseg;
    if (row >= p.rows || col >= p.cols) continue;
    const uint4 w = *reinterpret_cast<const uint4*>(p.X + row * p.ldx + col);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    uint32_t q[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      q[i] = cvt_e4m3x2(__fmul_rn(bf16_hi(ws[i]), inv), __fmul_rn(bf16_lo(ws[i]), inv));  // byte 0 = lower column
    if (p.transpose) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        tile[8 * cseg + 2 * i][rr] = static_cast<uint8_t>(q[i]);
        tile[8 * cseg + 2 * i + 1][rr] = static_cast<uint8_t>(q[i] >> 8);
      }
    } else {
      *reinterpret_cast<uint2*>(p.out + row * p.ldo + col) = make_uint2(q[0] | (q[1] << 16), q[2] | (q[3] << 16));
    }
  }
  if (!p.transpose) return;
  __syncthreads();
  // 64 output rows (columns of X) x 128 bytes: 8 threads of 16 bytes per row
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    const int cc = pass * 32 + (tid >> 3);
    const int seg = tid & 7;
    const int64_t orow = c0 + cc, ocol = r0 + 16 * seg;
    if (orow >= p.cols || ocol >= p.rows) continue;
    const uint4 v = *reinterpret_cast<const uint4*>(&tile[cc][16 * seg]);
    *reinterpret_cast<uint4*>(p.out + orow * p.ldo + ocol) = v;
  }
}

}  // namespace w4a4
