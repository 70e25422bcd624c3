// quant.cuh -- NVFP4 quantisation kernels.
//
//   amax_kernel         A = max |x * inv_s| over the tensor.  Grid-stride,
//                       16-byte loads, warp-shuffle + shared-memory block
//                       max, one partial maximum per CTA (no atomics, so the
//                       result is deterministic).
//   quant_kernel        the streaming quantise pass, tensor amax known:
//                       persistent, one CTA per SM walking (128-row block,
//                       K slice) work items; TMA streams 128 x 64 tiles of
//                       the source through one mbarrier ring (128-byte
//                       swizzle); thread t owns row t of the tile, so the
//                       four 16-element blocks of a 64-wide chunk are reduced
//                       without shuffles and its four scale bytes form one
//                       32-bit word of the SF atom.  With a low-rank factor,
//                       one elected thread feeds the same tiles to
//                       tcgen05.mma (kind::f16, M=128, N=r) so that U = X L1
//                       accumulates in TMEM; each K slice writes its fp32
//                       partial, and the last slice of a row block (ticket
//                       counter) sums the partials in slice order, scales by
//                       1/(t_x t_w) and writes the bf16 hi/lo pair.
//   quant_fused_kernel  the single pass: every tile of the activation stays
//                       resident in shared memory while a grid barrier
//                       reduces the tensor amax, then the same quantisation.
//
// Synchronisation words in the workspace: the per-row-block tickets are zero
// at rest (the last participant to read one clears it before its kernel
// ends); the single-pass grid barrier keeps a launch generation and, per
// generation parity, an arrival counter and a maximum word, the other
// parity's pair being cleared one launch ahead.  A call therefore needs no
// memset as long as the workspace was zeroed once before its first use.
//
// The quantiser follows the NVFP4 arithmetic stated in include/w4a4.h; every
// rounding step is an explicit correctly rounded fp32 intrinsic so that codes
// and scale bytes match a plain IEEE implementation bit for bit.
#pragma once

#include "sm100.cuh"

namespace w4a4 {

constexpr int kAmaxThreads = 256;
constexpr int kAmaxMaxBlocks = 1024;
constexpr int kQRows = 128;       // rows per CTA (one TMEM lane per row)
constexpr int kQChunk = 64;       // K elements per pipeline step (one SF atom column)
// Streaming quantiser (pass 2), persistent, one CTA per SM: three groups of
// four compute warps (one thread per row of the 128-row tile; group g takes
// the CTA's chunks g, g+3, ...), a TMA producer warp, the TMEM owner / U-MMA
// warp and four U warps (one per TMEM lane quarter).
constexpr int kQGroups = 3;
constexpr int kQComputeWarps = 4 * kQGroups;
constexpr int kQProducerWarp = kQComputeWarps;      // TMA producer
constexpr int kQMmaWarp = kQComputeWarps + 1;       // TMEM owner, issues the U = X L1 MMAs
constexpr int kQUWarp0 = kQComputeWarps + 2;        // four warps: partial U out, row-block sums
constexpr int kQThreads = 32 * (kQComputeWarps + 6);
constexpr int kQMaxSplits = 32;   // K slices per row block at most (each adds a partial U to sum)
constexpr int kQAcc = 4;          // U accumulators in TMEM: the MMAs run up to three items ahead of the U warps

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ------------------------------------------------------------------ pass 1
// The tensor amax of the smoothed activation, max |fl(x_mk * s_k)|.  Rounding
// is monotonic and s_k > 0, so it equals max over k of fl(max_m |x_mk| * s_k):
// each thread owns one 16-byte column segment (8 bf16 or 4 fp32 channels) of a
// band of rows, keeps the running column maxima of |x| (packed bf16x2 maxima
// for bf16) and multiplies by s once per column at the end.  A warp reads 512
// contiguous bytes of a row per load; every lane keeps kAmaxUnroll loads in
// flight.  Plain cached loads leave the tensor in L2 for pass 2.
constexpr int kAmaxUnroll = 8;


template <typename SrcT>
__global__ void __launch_bounds__(kAmaxThreads) amax_kernel(const SrcT* __restrict__ X, int64_t M,
                                                            int64_t K, int64_t ld,
                                                            const float* __restrict__ inv_s,
                                                            float* __restrict__ partials,
                                                            int rows_per_cta) {
  constexpr int EPV = 16 / sizeof(SrcT);  // channels per 16-byte segment
  const int lane = threadIdx.x & 31;
  const int64_t segs = K / EPV;
  const int64_t seg = static_cast<int64_t>(blockIdx.x) * kAmaxThreads + threadIdx.x;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_cta;
  const int64_t r1 = r0 + rows_per_cta < M ? r0 + rows_per_cta : M;
  float m = 0.0f;
  if (seg < segs) {
    const SrcT* col = X + seg * EPV;
    uint32_t acc[4] = {0u, 0u, 0u, 0u};  // |x| maxima: 4 bf16x2 words or 4 fp32 bit patterns
    for (int64_t row = r0; row < r1; row += kAmaxUnroll) {
      uint4 raw[kAmaxUnroll];
#pragma unroll
      for (int u = 0; u < kAmaxUnroll; ++u)
        if (row + u < r1) raw[u] = __ldg(reinterpret_cast<const uint4*>(col + (row + u) * ld));
#pragma unroll
      for (int u = 0; u < kAmaxUnroll; ++u) {
        if (row + u >= r1) continue;
        const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if constexpr (sizeof(SrcT) == 2)
            acc[j] = bf16x2_absmax(acc[j], w[j]);
          else
            acc[j] = __float_as_uint(fmaxf(__uint_as_float(acc[j]), fabsf(__uint_as_float(w[j]))));
        }
      }
    }
    float v[EPV];
    if constexpr (sizeof(SrcT) == 2) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[2 * j] = bf16_lo(acc[j] & 0x7FFF7FFFu);
        v[2 * j + 1] = bf16_hi(acc[j] & 0x7FFF7FFFu);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = __uint_as_float(acc[j]);
    }
    if (inv_s != nullptr) {
#pragma unroll
      for (int j = 0; j < EPV; j += 4) {
        const float4 s4 = __ldg(reinterpret_cast<const float4*>(inv_s + seg * EPV + j));
        v[j] = __fmul_rn(v[j], s4.x);
        v[j + 1] = __fmul_rn(v[j + 1], s4.y);
        v[j + 2] = __fmul_rn(v[j + 2], s4.z);
        v[j + 3] = __fmul_rn(v[j + 3], s4.w);
      }
    }
#pragma unroll
    for (int j = 0; j < EPV; ++j) m = fmaxf(m, v[j]);
  }
  __shared__ float red[kAmaxThreads / 32];
  m = warp_max(m);
  if (lane == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  const int cta = blockIdx.y * gridDim.x + blockIdx.x;
  if (threadIdx.x < 32) {
    float r = threadIdx.x < kAmaxThreads / 32 ? red[threadIdx.x] : 0.0f;
    r = warp_max(r);
    if (threadIdx.x == 0) partials[cta] = r;
  }
}

// ------------------------------------------------------------------ pass 2
struct QuantParams {
  int64_t M, K;
  const float* inv_s;      // [K] or nullptr
  const float* partials;   // pass-1 maxima
  int n_partials;
  const float* t_w;        // weight tensor scale (low-rank only)
  uint8_t* q;              // [M, K/2]
  uint8_t* sf;             // SF atom layout
  float* t_out;            // tensor scale (written by CTA (0,0))
  float* u_part;           // [splits][row_blocks*128][32] fp32 partial U
  __nv_bfloat16* u_out;    // [M, 64] hi|lo
  int* tickets;            // [row_blocks]
  int chunks_per_split;     // single-pass kernel: K slice of each CTA
  int splits;               // single-pass kernel: K slices per row block
  int row_blocks;
  int has_lr;
  int r;                   // low-rank rank (16 or 32) when has_lr
  int* status;
};

template <typename SrcT>
struct QuantTile {
  // bf16: one 128 x 64 box (16 KB); fp32: two 128 x 32 boxes (32 KB).
  static constexpr int kBytes = kQRows * kQChunk * static_cast<int>(sizeof(SrcT));
  static constexpr int kBoxes = sizeof(SrcT) / 2;
  static constexpr int kStages = sizeof(SrcT) == 2 ? 9 : 6;
  // The producer refills kGroup ring slots at once, so that the loads of
  // adjacent chunks of the same rows reach DRAM together.
  static constexpr int kGroup = 3;
  static constexpr int kL1Bytes = 32 * kQChunk * 2;  // L1t tile, 32 x 64 bf16 (4 KB)
  static constexpr int kL1Off = kBytes;
  static constexpr int kInvSOff = kBytes + (sizeof(SrcT) == 2 ? kL1Bytes : 0);  // 64 fp32 of inv_s
  static constexpr int kStageBytes = (kInvSOff + kQChunk * 4 + 1023) / 1024 * 1024;
  // ring, then per compute warp kCodeBufs 1 KB staging buffers for its codes
  // (32 rows x 32 bytes, written out by TMA), barriers + scalars (512 B), 1 KB
  // alignment slack
  static constexpr int kCodeBuf = 32 * 32;
  static constexpr int kCodeBufs = 2;
  static constexpr int kCodeOff = kStageBytes * kStages;
  // the code multiplier 1/(dec(e) t) of every scale code e (256 fp32)
  static constexpr int kRqOff = kCodeOff + kQComputeWarps * kCodeBufs * kCodeBuf;
  static constexpr int kBarOff = kRqOff + 256 * 4;
  static constexpr int kSmem = kBarOff + 512 + 1024;
  // full/empty/mma_done per stage, acc_full/acc_empty per accumulator, drain;
  // then the TMEM address, abort flag, per-warp maxima and the last-slice flag
  static_assert(8 * (3 * kStages + 2 * kQAcc + 1) + 4 * (2 + kQThreads / 32 + 1) <= 512, "barrier area");
  static_assert(kSmem <= 232448, "shared memory budget");
};

// Read 8 consecutive source elements [8c, 8c+8) of row ``r`` from a 128-byte
// swizzled tile (row pitch 128 bytes, 16-byte chunk index XOR row % 8).
template <typename SrcT>
__device__ __forceinline__ void load8(const uint8_t* tile, int r, int c, float (&v)[8]) {
  if constexpr (sizeof(SrcT) == 2) {
    const uint4 w = *reinterpret_cast<const uint4*>(tile + r * 128 + ((c ^ (r & 7)) << 4));
    v[0] = bf16_lo(w.x); v[1] = bf16_hi(w.x);
    v[2] = bf16_lo(w.y); v[3] = bf16_hi(w.y);
    v[4] = bf16_lo(w.z); v[5] = bf16_hi(w.z);
    v[6] = bf16_lo(w.w); v[7] = bf16_hi(w.w);
  } else {
    // fp32: elements 8c..8c+7 are 16-byte chunks 2c, 2c+1 of the row; box b
    // holds chunks [8b, 8b+8).
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int g = 2 * c + h;
      const uint8_t* box = tile + (g >> 3) * (kQRows * 128);
      const float4 w = *reinterpret_cast<const float4*>(box + r * 128 + (((g & 7) ^ (r & 7)) << 4));
      v[4 * h] = w.x; v[4 * h + 1] = w.y; v[4 * h + 2] = w.z; v[4 * h + 3] = w.w;
    }
  }
}

// Eight smoothed values of row ``r``, elements 8u..8u+7 of a resident chunk
// (``inv`` holds the chunk's 64 reciprocal smoothing factors).
template <typename SrcT>
__device__ __forceinline__ void load_unit(const uint8_t* tile, const float* inv, bool has_inv, int r, int u,
                                          float (&v)[8]) {
  load8<SrcT>(tile, r, u, v);
  if (has_inv) {
    const float4 s0 = reinterpret_cast<const float4*>(inv)[2 * u];
    const float4 s1 = reinterpret_cast<const float4*>(inv)[2 * u + 1];
    mul2_rn(v[0], v[1], v[0], v[1], s0.x, s0.y);
    mul2_rn(v[2], v[3], v[2], v[3], s0.z, s0.w);
    mul2_rn(v[4], v[5], v[4], v[5], s1.x, s1.y);
    mul2_rn(v[6], v[7], v[6], v[7], s1.z, s1.w);
  }
}

__device__ __forceinline__ float tensor_scale_from(float amax) {
  float t = __fdiv_rn(amax, 2688.0f);
  if (!(t >= 1.17549435e-38f)) t = 1.0f;  // not a normal number -> 1
  return t;
}

// Columns 16hh .. 16hh+15 of a row's low-rank sum, scaled by ra = 1/(t_x t_w),
// as the bf16 hi|lo pair (row of 2r bf16: hi in columns [0, r), lo in [r, 2r)).
__device__ __forceinline__ void store_lowrank16(const QuantParams& p, float ra, __nv_bfloat16* urow, int hh,
                                                const float (&acc)[16]) {
  uint32_t hi[8], lo[8];
#pragma unroll
  for (int j = 0; j < 16; j += 2) {
    const float a0 = __fmul_rn(acc[j], ra), a1 = __fmul_rn(acc[j + 1], ra);
    const uint32_t h = pack_bf16x2(a0, a1);
    hi[j / 2] = h;
    lo[j / 2] = pack_bf16x2(__fsub_rn(a0, bf16_lo(h)), __fsub_rn(a1, bf16_hi(h)));
  }
  uint4* dh = reinterpret_cast<uint4*>(urow + 16 * hh);
  uint4* dl = reinterpret_cast<uint4*>(urow + p.r + 16 * hh);
  dh[0] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
  dh[1] = make_uint4(hi[4], hi[5], hi[6], hi[7]);
  dl[0] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  dl[1] = make_uint4(lo[4], lo[5], lo[6], lo[7]);
}

// A row block covered by one piece: its U is final in TMEM; the row's sum is
// 0 + u (the same arithmetic as the sum of one partial), no round trip.
__device__ __forceinline__ void store_lowrank_row(const QuantParams& p, float ra, int64_t row,
                                                  const uint32_t (&u)[32]) {
  __nv_bfloat16* urow = p.u_out + row * 2 * p.r;
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {  // r = 16 or 32: one or two groups of 16 columns
    if (hh < p.r / 16) {
      float acc[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[j] = __fadd_rn(0.0f, __uint_as_float(u[16 * hh + j]));
      store_lowrank16(p, ra, urow, hh, acc);
    }
  }
}

// The last K slice of a row block sums the fp32 partials in slice order,
// scales by 1/(t_x t_w) and writes the bf16 hi|lo pair of its row (columns
// in groups of 16, two slices' loads in flight).
__device__ __forceinline__ void finalize_lowrank(const QuantParams& p, float t, int64_t rows_pad, int64_t prow,
                                                 int64_t row, int n_parts) {
  __threadfence();
  const float ra = __frcp_rn(__fmul_rn(t, __ldg(p.t_w)));
  __nv_bfloat16* urow = p.u_out + row * 2 * p.r;
#pragma unroll 1
  for (int hh = 0; hh < p.r / 16; ++hh) {
    float acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
    for (int sp0 = 0; sp0 < n_parts; sp0 += 2) {
      float4 w[2][4];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        if (sp0 + q < n_parts) {
          const float4* src = reinterpret_cast<const float4*>(
              p.u_part + (static_cast<int64_t>(sp0 + q) * rows_pad + prow) * 32 + 16 * hh);
#pragma unroll
          for (int j = 0; j < 4; ++j) w[q][j] = __ldcg(src + j);
        }
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        if (sp0 + q < n_parts) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc[4 * j] = __fadd_rn(acc[4 * j], w[q][j].x);
            acc[4 * j + 1] = __fadd_rn(acc[4 * j + 1], w[q][j].y);
            acc[4 * j + 2] = __fadd_rn(acc[4 * j + 2], w[q][j].z);
            acc[4 * j + 3] = __fadd_rn(acc[4 * j + 3], w[q][j].w);
          }
        }
      }
    }
    if (row < p.M) store_lowrank16(p, ra, urow, hh, acc);
  }
}

template <typename SrcT>
__global__ void __launch_bounds__(kQThreads, 1) quant_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                          const __grid_constant__ CUtensorMap tm_l1,
                                                          const __grid_constant__ CUtensorMap tm_q,
                                                          const QuantParams p) {
  using Tile = QuantTile<SrcT>;
  constexpr int S = Tile::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Tile::kBarOff);
  uint64_t* empty = full + S;
  uint64_t* mma_done = empty + S;
  uint64_t* acc_full = mma_done + S;              // [kQAcc] an item's U MMAs are complete
  uint64_t* acc_empty = acc_full + kQAcc;         // [kQAcc] the U warps have read the accumulator
  uint64_t* drain = acc_empty + kQAcc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(tmem_slot + 2);  // one float per warp
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2 + kQThreads / 32);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int chunks = static_cast<int>(p.K / kQChunk);
  const bool lr = p.has_lr != 0;
  grid_launch_dependents();

  // The (row block, chunk) sequence of the whole activation, row block by
  // row block, is cut into gridDim.x equal contiguous ranges, one per CTA.
  // A CTA's work items are the pieces of its range that lie in one row block
  // (rarely more than two); a row block is covered by the pieces of up to
  // ceil(gridDim / row_blocks) + 1 consecutive CTAs, whose partial U are
  // summed in CTA order.
  const int64_t total_chunks = static_cast<int64_t>(p.row_blocks) * chunks;
  const int64_t g_begin = static_cast<int64_t>(blockIdx.x) * total_chunks / gridDim.x;
  const int64_t g_end = static_cast<int64_t>(blockIdx.x + 1) * total_chunks / gridDim.x;
  auto cta_of = [&](int64_t g) {  // the CTA whose range holds chunk g
    return static_cast<int>(((g + 1) * gridDim.x - 1) / total_chunks);
  };
  struct Piece {
    int rb, kc0, n;
  };
  auto piece_at = [&](int64_t g) {  // the item of this CTA that starts at chunk g
    Piece pc;
    pc.rb = static_cast<int>(g / chunks);
    pc.kc0 = static_cast<int>(g - static_cast<int64_t>(pc.rb) * chunks);
    pc.n = static_cast<int>(min(g_end, static_cast<int64_t>(pc.rb + 1) * chunks) - g);
    return pc;
  };

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 4);  // the four warps of the group that took the chunk
      mbar_init(smem_u32(&mma_done[s]), 1);
    }
    for (int a = 0; a < kQAcc; ++a) {
      mbar_init(smem_u32(&acc_full[a]), 1);
      mbar_init(smem_u32(&acc_empty[a]), 4);  // the four U warps
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (lr && warp == kQMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 32 * kQAcc);  // 32-column U accumulators
    tmem_relinquish();
  }
  // set-up above may overlap the previous kernel (programmatic launch);
  // nothing below may touch memory before it has completed
  grid_dependency_wait();
  // tensor scale from the pass-1 partial maxima (the same value in every CTA)
  float m = 0.0f;
  for (int i = tid; i < p.n_partials; i += kQThreads) m = fmaxf(m, p.partials[i]);
  m = warp_max(m);
  if (lane == 0) red[warp] = m;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  float amax = red[0];
#pragma unroll
  for (int w = 1; w < kQThreads / 32; ++w) amax = fmaxf(amax, red[w]);
  const float t = tensor_scale_from(amax);
  const float rt = __frcp_rn(t);
  if (blockIdx.x == 0 && tid == 0) *p.t_out = t;
  const uint32_t tmem = lr ? *tmem_slot : 0u;
  // The code multiplier 1/(dec(e) t) of every scale code a block can get
  // (1..126: non-negative, saturated at 448); code 0 leaves the block's codes
  // +0 and never uses its entry.  The same correctly rounded values the
  // per-block computation gives, looked up instead of computed.
  float* rq_tab = reinterpret_cast<float*>(smem + Tile::kRqOff);
  if (tid < 256)
    rq_tab[tid] = (tid >= 1 && tid <= 126)
                      ? __frcp_rn(__fmul_rn(e4m3x2_to_f32(static_cast<uint32_t>(tid)).y, t))
                      : 0.0f;
  __syncthreads();

  if (warp == kQProducerWarp) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_x);
      if (lr) tma_prefetch_desc(&tm_l1);
      const uint32_t inv_bytes = p.inv_s != nullptr ? kQChunk * 4 : 0;
      const int total = static_cast<int>(g_end - g_begin);  // this CTA's chunks
      int c = 0;  // this CTA's chunks, in order
      bool ok = true;
      for (int64_t g = g_begin; g < g_end && ok; g += piece_at(g).n) {
        const Piece pc = piece_at(g);
        const int rb = pc.rb;
        const int kc0 = pc.kc0;
        const int n = pc.n;
        for (int i = 0; i < n; ++i, ++c) {
          const int s = c % S;
          if (c % Tile::kGroup == 0) {
            // a new group of chunks: wait until all of its slots are free, so
            // that its loads go out back to back
            const int c_end = min(c + Tile::kGroup, total);
            for (int j = max(c, S); j < c_end && ok; ++j) {
              const uint32_t ph = ((j / S) - 1) & 1;  // the fill of chunk j - S
              ok = mbar_wait(smem_u32(&empty[j % S]), ph, abort_flag, p.status) &&
                   (!lr || mbar_wait(smem_u32(&mma_done[j % S]), ph, abort_flag, p.status));
            }
            if (!ok) break;
          }
          const uint32_t bar = smem_u32(&full[s]);
          uint8_t* dst = smem + s * Tile::kStageBytes;
          const int kx = (kc0 + i) * kQChunk;
          if constexpr (sizeof(SrcT) == 2) {
            mbar_arrive_expect_tx(bar, Tile::kBytes + (lr ? 2 * kQChunk * p.r : 0) + inv_bytes);
            tma_load_2d(smem_u32(dst), &tm_x, bar, kx, rb * kQRows);
            if (lr) tma_load_2d(smem_u32(dst + Tile::kL1Off), &tm_l1, bar, kx, 0);
          } else {
            mbar_arrive_expect_tx(bar, Tile::kBytes + inv_bytes);
            tma_load_2d(smem_u32(dst), &tm_x, bar, kx, rb * kQRows);
            tma_load_2d(smem_u32(dst + kQRows * 128), &tm_x, bar, kx + 32, rb * kQRows);
          }
          if (inv_bytes) bulk_load(smem_u32(dst + Tile::kInvSOff), p.inv_s + kx, inv_bytes, bar);
        }
      }
      // every fill issued must land before the shared memory is released
      for (int j = max(0, c - S); j < c; ++j) mbar_wait_drain(smem_u32(&full[j % S]), (j / S) & 1);
    }
  } else if (warp == kQMmaWarp) {
    // ------------------------------------------------------- U = X L1 MMAs, one accumulator per item
    if (lr && lane == 0) {
      int c = 0, j = 0;
      bool ok = true;
      for (int64_t g = g_begin; g < g_end && ok; g += piece_at(g).n, ++j) {
        const int a = j % kQAcc;
        if (j >= kQAcc && !mbar_wait(smem_u32(&acc_empty[a]), ((j / kQAcc) - 1) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d = tmem + 32u * a;
        const int n = piece_at(g).n;
        for (int i = 0; i < n; ++i, ++c) {
          const int s = c % S;
          if (!mbar_wait(smem_u32(&full[s]), (c / S) & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + s * Tile::kStageBytes);
          const uint32_t b_base = a_base + Tile::kL1Off;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = smem_desc(a_base + 32 * k, 16, 1024, kSwizzle128B);
            const uint64_t bd = smem_desc(b_base + 32 * k, 16, 1024, kSwizzle128B);
            mma_bf16(d, ad, bd, idesc_bf16(128, p.r), (i > 0 || k > 0) ? 1u : 0u);
          }
          tc_commit(smem_u32(&mma_done[s]));
        }
        if (ok) tc_commit(smem_u32(&acc_full[a]));
      }
      // all MMAs of this thread complete before TMEM is released
      tc_commit(smem_u32(drain));
      mbar_wait_drain(smem_u32(drain), 0);
    }
  } else if (warp >= kQUWarp0) {
    // ------------------------------------------------------- partial U out; row-block sums
    if (lr) {
      const int quarter = warp & 3;  // the TMEM lane quarter this warp may read
      const int ut = (warp - kQUWarp0) * 32 + lane;
      const int64_t rows_pad = static_cast<int64_t>(p.row_blocks) * kQRows;
      const float ra_u = __frcp_rn(__fmul_rn(t, __ldg(p.t_w)));
      int j = 0;
      for (int64_t g = g_begin; g < g_end; g += piece_at(g).n, ++j) {
        const int a = j % kQAcc;
        const int rb = piece_at(g).rb;
        // this piece's place among the row block's pieces, and their number
        const int b0 = cta_of(static_cast<int64_t>(rb) * chunks);
        const int split = static_cast<int>(blockIdx.x) - b0;
        const int n_parts = cta_of(static_cast<int64_t>(rb + 1) * chunks - 1) - b0 + 1;
        if (!mbar_wait(smem_u32(&acc_full[a]), (j / kQAcc) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        uint32_t u[32];
        tmem_ld_32cols(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + 32u * a, u);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&acc_empty[a]));
        const int64_t prow = static_cast<int64_t>(rb) * kQRows + quarter * 32 + lane;
        if (n_parts == 1) {
          if (prow < p.M) store_lowrank_row(p, ra_u, prow, u);
          continue;
        }
        float4* dst = reinterpret_cast<float4*>(p.u_part + (static_cast<int64_t>(split) * rows_pad + prow) * 32);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          dst[q] = make_float4(__uint_as_float(u[4 * q]), __uint_as_float(u[4 * q + 1]),
                               __uint_as_float(u[4 * q + 2]), __uint_as_float(u[4 * q + 3]));
        __threadfence();
        named_bar_sync(2, 128);  // the four U warps' partial rows are out
        if (ut == 0) {
          const int ticket = atomicAdd(&p.tickets[rb], 1);
          const bool last = ticket == n_parts - 1;
          if (last) p.tickets[rb] = 0;  // every slice has taken its ticket
          *last_flag = last ? 1 : 0;
        }
        named_bar_sync(2, 128);
        if (*last_flag) {
          // this was the row block's last slice: sum every slice's partial
          // for row ut of the block, in slice order
          const int64_t frow = static_cast<int64_t>(rb) * kQRows + ut;
          finalize_lowrank(p, t, rows_pad, frow, frow, n_parts);
        }
      }
    }
  } else {
    // ------------------------------------------------------- quantise rows
    const bool has_inv = p.inv_s != nullptr;
    if (lane == 0) tma_prefetch_desc(&tm_q);
    // this warp's 32 rows of codes go out through kCodeBufs staging buffers
    uint8_t* code_stage = smem + Tile::kCodeOff + warp * Tile::kCodeBufs * Tile::kCodeBuf;
    int n_stored = 0;
    const int grp = warp >> 2;
    const int row_in_tile = tid & (kQRows - 1);
    const int total = static_cast<int>(g_end - g_begin);
    for (int c = grp; c < total; c += kQGroups) {
      const int64_t g = g_begin + c;  // chunk c of this CTA in the whole sequence
      const int rb = static_cast<int>(g / chunks);
      const int kc = static_cast<int>(g - static_cast<int64_t>(rb) * chunks);
      const int s = c % S;
      if (!mbar_wait(smem_u32(&full[s]), (c / S) & 1, abort_flag, p.status)) break;
      const uint8_t* tile = smem + s * Tile::kStageBytes;
      const float* inv = reinterpret_cast<const float*>(tile + Tile::kInvSOff);
      uint32_t cw[8];
      uint32_t e4 = 0u;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // blocks 2h and 2h+1 (elements 32h .. 32h+31 of the chunk)
        float x[32];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          load_unit<SrcT>(tile, inv, has_inv, row_in_tile, 4 * h + u, *reinterpret_cast<float(*)[8]>(&x[8 * u]));
        const float bm0 = absmax16(x), bm1 = absmax16(x + 16);
        // both blocks' scale bytes in one conversion; byte 0 = block 2h
        const uint32_t e2 = cvt_e4m3x2(div6(__fmul_rn(bm1, rt)), div6(__fmul_rn(bm0, rt))) & 0xFFFFu;
        e4 |= e2 << (16 * h);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const uint32_t e = (e2 >> (8 * q)) & 0xFFu;
          const float rq = rq_tab[e];  // 1/(dec(e) t)
#pragma unroll
          for (int uu = 0; uu < 2; ++uu) {
            float v[8];
#pragma unroll
            for (int jj = 0; jj < 8; jj += 2)
              mul2_rn(v[jj], v[jj + 1], x[16 * q + 8 * uu + jj], x[16 * q + 8 * uu + jj + 1], rq, rq);
            // a zero scale leaves the block's codes +0 (masked, not branched)
            cw[4 * h + 2 * q + uu] = e != 0u ? cvt_e2m1x8(v) : 0u;
          }
        }
      }
      // Every value read from the stage has been consumed: release it (the
      // shared-memory reads are ordered before the refill's TMA writes by the
      // proxy fence and the barrier's release/acquire).
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
      // codes: row ``lane`` of the warp's 32 rows, 32 bytes, into a staging
      // buffer whose last TMA store (kCodeBufs chunks of this warp ago) has
      // finished reading it; lanes with bit 2 set store their halves in the
      // other order (no bank conflicts); the TMA store drops rows >= M
      uint8_t* cb = code_stage + (n_stored % Tile::kCodeBufs) * Tile::kCodeBuf;
      if (n_stored >= Tile::kCodeBufs) {
        if (lane == 0) bulk_wait_group_read<Tile::kCodeBufs - 1>();
        __syncwarp();
      }
      const int first = (lane >> 2) & 1;
      *reinterpret_cast<uint4*>(cb + lane * 32 + 16 * first) =
          first ? make_uint4(cw[4], cw[5], cw[6], cw[7]) : make_uint4(cw[0], cw[1], cw[2], cw[3]);
      *reinterpret_cast<uint4*>(cb + lane * 32 + 16 * (first ^ 1)) =
          first ? make_uint4(cw[0], cw[1], cw[2], cw[3]) : make_uint4(cw[4], cw[5], cw[6], cw[7]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&tm_q, smem_u32(cb), kc * 32, rb * kQRows + (warp & 3) * 32);
        bulk_commit_group();
      }
      ++n_stored;
      const int64_t atom = static_cast<int64_t>(rb) * chunks + kc;
      *reinterpret_cast<uint32_t*>(p.sf + atom * 512 + (row_in_tile & 31) * 16 + (row_in_tile >> 5) * 4) = e4;
    }
    // the code stores have landed before the CTA ends
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  }

  // Every role has finished (or given up); in-flight copies and MMAs drained.
  tc_fence_before();
  __syncthreads();
  if (lr && warp == kQMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 32 * kQAcc);
  }
}

// ------------------------------------------------------------------ layout helper
// SF atoms -> row-major [rows, K/16]: one thread per (row, 64-wide K group);
// the group's four scale bytes of a row are one 32-bit word of its atom.
__global__ void sf_to_rowmajor_kernel(const uint8_t* __restrict__ atoms, int64_t rows, int64_t groups,
                                      uint8_t* __restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= rows * groups) return;
  const int64_t m = i / groups, g = i % groups;
  const uint32_t w = *reinterpret_cast<const uint32_t*>(atoms + ((m / kQRows) * groups + g) * 512 + (m % 32) * 16 +
                                                         ((m / 32) % 4) * 4);
  *reinterpret_cast<uint32_t*>(out + (m * groups + g) * 4) = w;
}

// ------------------------------------------------------------------ fused single pass
// When every (128-row block, K slice) tile of the activation fits in the
// shared memory of one co-resident wave of CTAs (one CTA per SM, up to
// kFusedMaxChunks 64-wide chunks each), the activation is read from HBM once:
// each CTA TMA-loads all of its chunks and keeps them resident, reduces its
// partial amax, meets every other CTA at a grid barrier (cooperative launch,
// bounded spin), then quantises from shared memory.  The U = X L1 MMAs run as
// the chunks land (L1t streams through a small ring).
constexpr int kFusedMaxChunks = 12;
constexpr int kFusedL1Ring = 7;  // L1t tiles in flight: as many as fit beside the resident X
constexpr int kFusedSlicesForSpread = 16;
// Grid barrier words in the workspace (32-bit word offsets, each on its own
// 128-byte line): the launch generation, two arrival counters and two
// tensor-maximum words (one of each per generation parity).
constexpr int kBarGen = 0;
constexpr int kBarCount = 32;   // + 32 * parity
constexpr int kBarAmax = 96;    // + 32 * parity
constexpr int kBarWords = 160;

struct FusedQuantSmem {
  static constexpr int kXBytes = kFusedMaxChunks * kQRows * kQChunk * 2;   // 192 KB
  static constexpr int kL1Bytes = kFusedL1Ring * 32 * kQChunk * 2;         // 28 KB
  static constexpr int kInvBytes = kFusedMaxChunks * kQChunk * 4;          // 3 KB
  static constexpr int kRqBytes = 256 * 4;                                 // 1/(dec(e) t) per scale code
  static constexpr int kBarBytes = 512;
  static constexpr int kBytes = kXBytes + kL1Bytes + kInvBytes + kRqBytes + kBarBytes + 1024;
  static_assert(kBytes <= 232448, "shared memory budget");
};

// Fused kernel roles (16 warps).  Warps 0-11 compute in three groups of four:
// group g owns chunks g, g+3, g+6, g+9 of the slice and thread (g, r) row r of
// each.  Warp 12 is the TMA producer and warp 13 the TMEM owner and U-MMA
// issuer; after that, warps 12-15 (one per TMEM lane quarter) move the partial
// U out of TMEM and, once every slice of the row block has its partial out
// (a per-row-block ticket), sum the partials of this CTA's share of the rows.
// The compute warps never wait for them.
constexpr int kFGroups = 3;
constexpr int kFComputeWarps = 4 * kFGroups;
constexpr int kFChunksPerThread = kFusedMaxChunks / kFGroups;
constexpr int kFProducerWarp = 12;
constexpr int kFMmaWarp = 13;
constexpr int kFUWarp0 = 12;  // warps 12-15 cover TMEM lane quarters 0-3
constexpr int kFThreads = 32 * 16;
static_assert(kFusedMaxChunks % kFGroups == 0, "chunk groups");
static_assert(kFComputeWarps * 32 >= 256, "one thread per scale code fills the multiplier table");

static_assert(kFUWarp0 % 4 == 0 && kFThreads == 32 * (kFUWarp0 + 4), "lane quarters");

// The grid barrier.  Every launch reads the generation G and uses the
// counter and maximum word of parity G & 1: each CTA folds its maximum into
// the word (atomic max; non-negative floats order as their bit patterns),
// then adds one to the counter with release semantics, and waits until the
// counter shows every CTA.  Block 0 then clears the other parity's two words
// for the next launch and advances G; the words of this launch's parity stay
// as they are until the launch after next clears them, so no CTA waits for a
// second round of atomics to learn that everyone has read the maximum.

__device__ __forceinline__ unsigned ld_relaxed_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_gpu(unsigned* p, unsigned v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded spin until a global counter reaches ``target``; false on timeout
// (then the abort flag and the device status are set).
__device__ __forceinline__ bool spin_until(const unsigned* ctr, unsigned target, volatile int* abort, int* status) {
  const long long start = clock64();
  while (ld_acquire_gpu(ctr) < target) {
    if (*abort) return false;
    if (clock64() - start > c_wait_bound_cycles) {
      *abort = 1;
      if (status) atomicExch(status, kStatusTimeout);
      return false;
    }
    __nanosleep(64);
  }
  return true;
}

__global__ void __launch_bounds__(kFThreads, 1)
    quant_fused_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_l1,
                       const __grid_constant__ CUtensorMap tm_q, const QuantParams p, unsigned* tickets,
                       unsigned* barrier) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xs = smem;
  uint8_t* l1s = smem + FusedQuantSmem::kXBytes;
  float* invs = reinterpret_cast<float*>(l1s + FusedQuantSmem::kL1Bytes);
  float* rq_tab = invs + kFusedMaxChunks * kQChunk;
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(rq_tab) + FusedQuantSmem::kRqBytes);
  uint64_t* l1_full = full + kFusedMaxChunks;
  uint64_t* l1_empty = l1_full + kFusedL1Ring;
  uint64_t* drain = l1_empty + kFusedL1Ring;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(tmem_slot + 2);  // kFComputeWarps floats
  float* t_shared = reinterpret_cast<float*>(tmem_slot + 2 + kFComputeWarps);
  unsigned* gen_shared = tmem_slot + 3 + kFComputeWarps;
  // tickets[rb] (zero at rest): slices of the row block whose partial U is
  // out, then slices that have seen them all; the last clears it.

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int rb = blockIdx.x / p.splits;
  const int split = blockIdx.x % p.splits;
  const int chunks = static_cast<int>(p.K / kQChunk);
  const int kc0 = split * p.chunks_per_split;
  const int kc1 = min(kc0 + p.chunks_per_split, chunks);
  const int n = kc1 - kc0;
  const bool lr = p.has_lr != 0;
  const bool has_inv = p.inv_s != nullptr;
  const int64_t rows_pad = static_cast<int64_t>(p.row_blocks) * kQRows;
  grid_launch_dependents();  // all CTAs are resident (cooperative launch)

  if (tid == 0) {
    for (int c = 0; c < kFusedMaxChunks; ++c) mbar_init(smem_u32(&full[c]), 1);
    for (int r = 0; r < kFusedL1Ring; ++r) {
      mbar_init(smem_u32(&l1_full[r]), 1);
      mbar_init(smem_u32(&l1_empty[r]), 1);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (lr && warp == kFMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = lr ? *tmem_slot : 0u;
  // set-up above may overlap the previous kernel (programmatic launch);
  // nothing below may touch memory before it has completed
  grid_dependency_wait();
  if (tid == 0) *gen_shared = ld_relaxed_gpu(barrier + kBarGen);

  float bmax[4 * kFChunksPerThread];  // compute threads: block maxima of their row
  const int r = tid & (kQRows - 1);
  const int grp = warp >> 2;

  if (warp >= kFUWarp0) {
    if (warp == kFProducerWarp && lane == 0) {
      // ---------------------------------------------------- all loads up front
      // Each chunk's L1t tile is queued right behind its X tile (while ring
      // slots last), so the U MMAs follow the chunks as they land; the
      // remaining L1t tiles reuse slots as the MMAs free them.
      tma_prefetch_desc(&tm_x);
      if (lr) tma_prefetch_desc(&tm_l1);
      auto load_l1 = [&](int c) {
        const int s = c % kFusedL1Ring;
        const uint32_t bar = smem_u32(&l1_full[s]);
        mbar_arrive_expect_tx(bar, p.r * kQChunk * 2);
        tma_load_2d(smem_u32(l1s + s * 32 * kQChunk * 2), &tm_l1, bar, (kc0 + c) * kQChunk, 0);
      };
      for (int c = 0; c < n; ++c) {
        const int kx = (kc0 + c) * kQChunk;
        const uint32_t bar = smem_u32(&full[c]);
        const uint32_t inv_bytes = has_inv ? kQChunk * 4 : 0;
        mbar_arrive_expect_tx(bar, kQRows * kQChunk * 2 + inv_bytes);
        tma_load_2d(smem_u32(xs + c * kQRows * kQChunk * 2), &tm_x, bar, kx, rb * kQRows);
        if (inv_bytes) bulk_load(smem_u32(invs + c * kQChunk), p.inv_s + kx, inv_bytes, bar);
        if (lr && c < kFusedL1Ring) load_l1(c);
      }
      if (lr) {
        for (int c = kFusedL1Ring; c < n; ++c) {
          const int s = c % kFusedL1Ring;
          if (!mbar_wait(smem_u32(&l1_empty[s]), ((c / kFusedL1Ring) - 1) & 1, abort_flag, p.status)) break;
          load_l1(c);
        }
      }
    } else if (warp == kFMmaWarp && lane == 0 && lr) {
      // ---------------------------------------------------- U = X L1 as the chunks land
      for (int c = 0; c < n; ++c) {
        const int s = c % kFusedL1Ring;
        if (!mbar_wait(smem_u32(&full[c]), 0, abort_flag, p.status)) break;
        if (!mbar_wait(smem_u32(&l1_full[s]), (c / kFusedL1Ring) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(xs + c * kQRows * kQChunk * 2);
        const uint32_t b_base = smem_u32(l1s + s * 32 * kQChunk * 2);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t ad = smem_desc(a_base + 32 * k, 16, 1024, kSwizzle128B);
          const uint64_t bd = smem_desc(b_base + 32 * k, 16, 1024, kSwizzle128B);
          mma_bf16(tmem, ad, bd, idesc_bf16(128, p.r), (c > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(smem_u32(&l1_empty[s]));
      }
      tc_commit(smem_u32(drain));
    }
    __syncwarp();
    if (lr) {
      // ------------------------------------------------------ partial U out of TMEM
      const int quarter = warp - kFUWarp0;
      uint32_t u[32];
      const bool ok = mbar_wait(smem_u32(drain), 0, abort_flag, p.status);
      __syncwarp();
      tc_fence_after();
      tmem_ld_32cols(tmem + (static_cast<uint32_t>(quarter * 32) << 16), u);
      tmem_ld_wait();
      if (!ok || n == 0) {
#pragma unroll
        for (int j = 0; j < 32; ++j) u[j] = 0u;
      }
      const int64_t prow = static_cast<int64_t>(rb) * kQRows + quarter * 32 + lane;
      float4* dst = reinterpret_cast<float4*>(p.u_part + (static_cast<int64_t>(split) * rows_pad + prow) * 32);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        dst[j] = make_float4(__uint_as_float(u[4 * j]), __uint_as_float(u[4 * j + 1]),
                             __uint_as_float(u[4 * j + 2]), __uint_as_float(u[4 * j + 3]));
      __threadfence();
      tc_fence_before();
      named_bar_sync(3, 128);  // the four U warps: TMEM read, partial out
      if (warp == kFMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 32);
      }
      if (tid == 32 * kFUWarp0) red_release_add(tickets + rb, 1u);
      // ---------------------------------------------------- wait for the tensor scale
      named_bar_sync(2, kFThreads);
      {
        // the four U warps meet at barrier 3 whatever the abort flag says
        if (tid == 32 * kFUWarp0 && !*abort_flag &&
            spin_until(tickets + rb, static_cast<unsigned>(p.splits), abort_flag, p.status) &&
            atom_acq_rel_add(tickets + rb, 1u) == 2u * static_cast<unsigned>(p.splits) - 1u)
          tickets[rb] = 0u;  // every slice has passed
        named_bar_sync(3, 128);
        if (!*abort_flag) {
          // -------------------------------------------------- this CTA's share of the U rows
          // The slices of a row block split its 128 rows; four threads per
          // row, eight columns each (r / 8 of them busy); the sum runs in
          // slice order.
          const float t = *t_shared;
          const int ut = tid - 32 * kFUWarp0;
          const int cg = ut & 3;
          const int rows_per = (kQRows + p.splits - 1) / p.splits;
          const int r_end = min(kQRows, (split + 1) * rows_per);
          const float ra = __frcp_rn(__fmul_rn(t, __ldg(p.t_w)));
          for (int rr = split * rows_per + (ut >> 2); cg < p.r / 8 && rr < r_end; rr += 32) {
            const int64_t prow2 = static_cast<int64_t>(rb) * kQRows + rr;
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
            for (int sp0 = 0; sp0 < p.splits; sp0 += 4) {
              float4 w[4][2];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                if (sp0 + q < p.splits) {
                  const float4* src = reinterpret_cast<const float4*>(
                      p.u_part + (static_cast<int64_t>(sp0 + q) * rows_pad + prow2) * 32 + cg * 8);
                  w[q][0] = __ldcg(src);
                  w[q][1] = __ldcg(src + 1);
                }
              }
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                if (sp0 + q < p.splits) {
#pragma unroll
                  for (int hh = 0; hh < 2; ++hh) {
                    acc[4 * hh] = __fadd_rn(acc[4 * hh], w[q][hh].x);
                    acc[4 * hh + 1] = __fadd_rn(acc[4 * hh + 1], w[q][hh].y);
                    acc[4 * hh + 2] = __fadd_rn(acc[4 * hh + 2], w[q][hh].z);
                    acc[4 * hh + 3] = __fadd_rn(acc[4 * hh + 3], w[q][hh].w);
                  }
                }
              }
            }
            if (prow2 < p.M) {
              uint32_t hi[4], lo[4];
#pragma unroll
              for (int j = 0; j < 8; j += 2) {
                const float a0 = __fmul_rn(acc[j], ra), a1 = __fmul_rn(acc[j + 1], ra);
                const uint32_t hb = pack_bf16x2(a0, a1);
                hi[j / 2] = hb;
                lo[j / 2] = pack_bf16x2(__fsub_rn(a0, bf16_lo(hb)), __fsub_rn(a1, bf16_hi(hb)));
              }
              __nv_bfloat16* urow = p.u_out + prow2 * 2 * p.r;
              *reinterpret_cast<uint4*>(urow + cg * 8) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
              *reinterpret_cast<uint4*>(urow + p.r + cg * 8) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------ phase A: block maxima
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < kFChunksPerThread; ++i) {
      const int c = grp + kFGroups * i;
#pragma unroll
      for (int b = 0; b < 4; ++b) bmax[4 * i + b] = 0.0f;
      if (c < n && mbar_wait(smem_u32(&full[c]), 0, abort_flag, p.status)) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          float v[8];
          load_unit<__nv_bfloat16>(xs + c * kQRows * kQChunk * 2, invs + c * kQChunk, has_inv, r, u, v);
          // |v| maxima as a tree, then into the block's running maximum
          const float m01 = fmaxf(fabsf(v[0]), fabsf(v[1])), m23 = fmaxf(fabsf(v[2]), fabsf(v[3]));
          const float m45 = fmaxf(fabsf(v[4]), fabsf(v[5])), m67 = fmaxf(fabsf(v[6]), fabsf(v[7]));
          bmax[4 * i + u / 2] = fmaxf(bmax[4 * i + u / 2], fmaxf(fmaxf(m01, m23), fmaxf(m45, m67)));
        }
#pragma unroll
        for (int b = 0; b < 4; ++b) m = fmaxf(m, bmax[4 * i + b]);
      }
    }
    m = warp_max(m);
    if (lane == 0) red[warp] = m;

    // ------------------------------------------------------ grid barrier (compute warps)
    named_bar_sync(1, 32 * kFComputeWarps);
    if (tid == 0) {
      float a = red[0];
#pragma unroll
      for (int w = 1; w < kFComputeWarps; ++w) a = fmaxf(a, red[w]);
      const unsigned g = *gen_shared;
      unsigned* count = barrier + kBarCount + 32 * (g & 1u);
      unsigned* amax_bits = barrier + kBarAmax + 32 * (g & 1u);
      atomicMax(amax_bits, __float_as_uint(a));
      red_release_add(count, 1u);  // orders the maximum before the arrival
      if (spin_until(count, gridDim.x, abort_flag, p.status)) {
        const float t = tensor_scale_from(__uint_as_float(ld_relaxed_gpu(amax_bits)));
        *t_shared = t;
        if (blockIdx.x == 0) *p.t_out = t;
      }
      if (blockIdx.x == 0) {
        // Once the counter shows every CTA, every CTA has read G (its arrival
        // used it).  After a timeout some CTA may not have arrived yet and
        // may still arrive on this parity: the words are then left
        // inconsistent, the status word says so, and the caller zeroes the
        // workspace before its next use.
        st_relaxed_gpu(barrier + kBarCount + 32 * ((g + 1u) & 1u), 0u);
        st_relaxed_gpu(barrier + kBarAmax + 32 * ((g + 1u) & 1u), 0u);
        st_relaxed_gpu(barrier + kBarGen, g + 1u);
      }
    }
    named_bar_sync(1, 32 * kFComputeWarps);
    if (lr) named_bar_arrive(2, kFThreads);  // the tensor scale is out for the U warps
    const float t = *t_shared;

    // ------------------------------------------------------ phase B: scales and codes
    // The code multiplier 1/(dec(e) t) of every scale code a block can get
    // (1..126: non-negative, saturated at 448), once per CTA.  Code 0 leaves
    // the block's codes +0 (its entry is never used); skipping it and the
    // codes above 126 keeps every reciprocal on the fast path (with them,
    // the table took 0.55 us instead of 0.16).
    if (tid < 256)
      rq_tab[tid] = (tid >= 1 && tid <= 126)
                        ? __frcp_rn(__fmul_rn(e4m3x2_to_f32(static_cast<uint32_t>(tid)).y, t))
                        : 0.0f;
    named_bar_sync(1, 32 * kFComputeWarps);
    // after the last named barrier of the compute warps: a warp that leaves
    // here never leaves another waiting at a barrier
    if (*abort_flag) return;
    const float rt = __frcp_rn(t);
    // Codes leave through TMA stores of the warp's 32 rows x 32 bytes, staged
    // in the first kilobyte of the warp's own rows of the chunk it has just
    // read.  The U MMAs read those tiles too: they are all complete once the
    // drain barrier has fired (long before this point).
    if (lr && !mbar_wait(smem_u32(drain), 0, abort_flag, p.status)) return;
    if (lane == 0) tma_prefetch_desc(&tm_q);
    // Every scale byte of the thread first (sixteen independent chains; the
    // scale words go out at once) with its code multiplier kept in a
    // register, then the codes chunk by chunk: no code waits on a table
    // lookup.
    uint32_t e4[kFChunksPerThread];
    float rq[4 * kFChunksPerThread];
#pragma unroll
    for (int i = 0; i < kFChunksPerThread; ++i) {
      // two blocks' scale bytes per conversion; byte b = block b
      const uint32_t lo = cvt_e4m3x2(div6(__fmul_rn(bmax[4 * i + 1], rt)), div6(__fmul_rn(bmax[4 * i], rt)));
      const uint32_t hi = cvt_e4m3x2(div6(__fmul_rn(bmax[4 * i + 3], rt)), div6(__fmul_rn(bmax[4 * i + 2], rt)));
      e4[i] = (lo & 0xFFFFu) | (hi << 16);
#pragma unroll
      for (int b = 0; b < 4; ++b) rq[4 * i + b] = rq_tab[(e4[i] >> (8 * b)) & 0xFFu];
      const int c = grp + kFGroups * i;
      if (c < n) {
        const int64_t atom = static_cast<int64_t>(rb) * chunks + kc0 + c;
        *reinterpret_cast<uint32_t*>(p.sf + atom * 512 + (r & 31) * 16 + (r >> 5) * 4) = e4[i];
      }
    }
#pragma unroll
    for (int i = 0; i < kFChunksPerThread; ++i) {
      const int c = grp + kFGroups * i;
      if (c < n) {
        const int kc = kc0 + c;
        uint32_t cw[8];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          // a zero scale leaves the block's codes +0 (computed anyway and
          // masked: no branch keeps the loads from moving up)
          const bool zero = ((e4[i] >> (8 * b)) & 0xFFu) == 0u;
#pragma unroll
          for (int uu = 0; uu < 2; ++uu) {
            float v[8];
            load_unit<__nv_bfloat16>(xs + c * kQRows * kQChunk * 2, invs + c * kQChunk, has_inv, r, 2 * b + uu, v);
            const float m = rq[4 * i + b];
            mul2_rn(v[0], v[1], v[0], v[1], m, m);
            mul2_rn(v[2], v[3], v[2], v[3], m, m);
            mul2_rn(v[4], v[5], v[4], v[5], m, m);
            mul2_rn(v[6], v[7], v[6], v[7], m, m);
            const uint32_t c8 = cvt_e2m1x8(v);
            cw[2 * b + uu] = zero ? 0u : c8;
          }
        }
        // every lane has read its rows of the chunk: stage this warp's codes
        // (row ``lane`` of 32, 32 bytes; lanes with bit 2 set store their
        // halves in the other order, no bank conflicts) and store them; the
        // TMA store drops rows >= M
        __syncwarp();
        uint8_t* cb = xs + c * kQRows * kQChunk * 2 + (warp & 3) * 32 * kQChunk * 2;
        const int first = (lane >> 2) & 1;
        *reinterpret_cast<uint4*>(cb + lane * 32 + 16 * first) =
            first ? make_uint4(cw[4], cw[5], cw[6], cw[7]) : make_uint4(cw[0], cw[1], cw[2], cw[3]);
        *reinterpret_cast<uint4*>(cb + lane * 32 + 16 * (first ^ 1)) =
            first ? make_uint4(cw[0], cw[1], cw[2], cw[3]) : make_uint4(cw[4], cw[5], cw[6], cw[7]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_q, smem_u32(cb), kc * 32, rb * kQRows + (warp & 3) * 32);
          bulk_commit_group();
        }
      }
    }
    // the code stores have landed before the CTA ends
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  }
  if (warp == kFProducerWarp && lane == 0) {
    // no copy may still be landing when the CTA exits
    for (int c = 0; c < n; ++c) mbar_wait_drain(smem_u32(&full[c]), 0);
  }
}

}  // namespace w4a4
