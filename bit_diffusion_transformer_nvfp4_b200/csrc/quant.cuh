// quant.cuh -- NVFP4 quantisation kernels.
//
//   amax_kernel   pass 1: A = max |x * inv_s| over the tensor.  Grid-stride,
//                 16-byte loads, warp-shuffle + shared-memory block max, one
//                 partial maximum per CTA (no atomics, so the result is
//                 deterministic).  Also clears the per-row-block tickets that
//                 pass 2 uses.
//   quant_kernel  pass 2: one CTA per (128-row block, K slice).  TMA streams
//                 128 x 64 tiles of the source through a 4-stage mbarrier
//                 ring (128-byte swizzle); thread t owns row t of the tile,
//                 so the four 16-element blocks of a 64-wide chunk are
//                 reduced without shuffles and its four scale bytes form one
//                 32-bit word of the SF atom.  When a low-rank factor is
//                 given, one elected thread feeds the same shared-memory
//                 tile to tcgen05.mma (kind::f16, M=128, N=r=32) so that
//                 U = X L1 accumulates in TMEM; each K slice writes its fp32
//                 partial, and the last slice of a row block (ticket counter)
//                 sums the partials in slice order, scales by 1/(t_x t_w) and
//                 writes the bf16 hi/lo pair.
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
constexpr int kQComputeWarps = 4;  // one thread per row of the 128-row tile
constexpr int kQProducerWarp = 4;  // TMA producer
constexpr int kQMmaWarp = 5;       // TMEM owner, issues the U = X L1 MMAs
constexpr int kQThreads = 32 * 6;
constexpr int kQTargetCtas = 296; // two CTAs per SM on a 148-SM part

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ------------------------------------------------------------------ pass 1
template <typename SrcT>
__global__ void __launch_bounds__(kAmaxThreads) amax_kernel(const SrcT* __restrict__ X, int64_t M,
                                                            int64_t K, int64_t ld,
                                                            const float* __restrict__ inv_s,
                                                            float* __restrict__ partials,
                                                            int* __restrict__ tickets,
                                                            int n_tickets) {
  constexpr int EPV = 16 / sizeof(SrcT);  // elements per 16-byte vector
  const int64_t vec_per_row = K / EPV;
  const int64_t total = M * vec_per_row;
  float m = 0.0f;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  auto absmax_vec = [&](int64_t i, const uint4 raw) {
    const int64_t row = i / vec_per_row;
    const int64_t col = (i - row * vec_per_row) * EPV;
    float v[EPV];
    if constexpr (sizeof(SrcT) == 2) {
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[2 * j] = bf16_lo(w[j]);
        v[2 * j + 1] = bf16_hi(w[j]);
      }
    } else {
      v[0] = __uint_as_float(raw.x);
      v[1] = __uint_as_float(raw.y);
      v[2] = __uint_as_float(raw.z);
      v[3] = __uint_as_float(raw.w);
    }
    if (inv_s != nullptr) {
#pragma unroll
      for (int j = 0; j < EPV; j += 4) {
        const float4 s = __ldg(reinterpret_cast<const float4*>(inv_s + col + j));
        v[j] = __fmul_rn(v[j], s.x);
        v[j + 1] = __fmul_rn(v[j + 1], s.y);
        v[j + 2] = __fmul_rn(v[j + 2], s.z);
        v[j + 3] = __fmul_rn(v[j + 3], s.w);
      }
    }
#pragma unroll
    for (int j = 0; j < EPV; ++j) m = fmaxf(m, fabsf(v[j]));
  };
  auto load = [&](int64_t i) {
    const int64_t row = i / vec_per_row;
    const int64_t col = (i - row * vec_per_row) * EPV;
    return __ldcs(reinterpret_cast<const uint4*>(X + row * ld + col));
  };
  int64_t i = i0;
  // four independent 16-byte loads in flight per thread
  for (; i + 3 * stride < total; i += 4 * stride) {
    const uint4 a = load(i), b = load(i + stride), c = load(i + 2 * stride), d = load(i + 3 * stride);
    absmax_vec(i, a);
    absmax_vec(i + stride, b);
    absmax_vec(i + 2 * stride, c);
    absmax_vec(i + 3 * stride, d);
  }
  for (; i < total; i += stride) absmax_vec(i, load(i));
  __shared__ float red[kAmaxThreads / 32];
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < kAmaxThreads / 32 ? red[threadIdx.x] : 0.0f;
    v = warp_max(v);
    if (threadIdx.x == 0) partials[blockIdx.x] = v;
  }
  if (blockIdx.x == 0) {
    for (int t = threadIdx.x; t < n_tickets; t += blockDim.x) tickets[t] = 0;
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
  int chunks_per_split;
  int splits;
  int has_lr;
  int* status;
};

template <typename SrcT>
struct QuantTile {
  // bf16: one 128 x 64 box (16 KB); fp32: two 128 x 32 boxes (32 KB).
  static constexpr int kBytes = kQRows * kQChunk * static_cast<int>(sizeof(SrcT));
  static constexpr int kBoxes = sizeof(SrcT) / 2;
  static constexpr int kStages = sizeof(SrcT) == 2 ? 4 : 3;
  static constexpr int kL1Bytes = 32 * kQChunk * 2;  // L1t tile, 32 x 64 bf16 (4 KB)
  static constexpr int kL1Off = kBytes;
  static constexpr int kInvSOff = kBytes + (sizeof(SrcT) == 2 ? kL1Bytes : 0);  // 64 fp32 of inv_s
  static constexpr int kStageBytes = (kInvSOff + kQChunk * 4 + 1023) / 1024 * 1024;
  static constexpr int kSmem = kStageBytes * kStages + 1024 + 256;
  static_assert(kStageBytes * kStages + 8 * (3 * kStages + 1) + 64 <= kStageBytes * kStages + 256, "barrier area");
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

__device__ __forceinline__ float tensor_scale_from(float amax) {
  float t = __fdiv_rn(amax, 2688.0f);
  if (!(t >= 1.17549435e-38f)) t = 1.0f;  // not a normal number -> 1
  return t;
}

template <typename SrcT>
__global__ void __launch_bounds__(kQThreads, 2) quant_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                          const __grid_constant__ CUtensorMap tm_l1,
                                                          const QuantParams p) {
  using Tile = QuantTile<SrcT>;
  constexpr int S = Tile::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Tile::kStageBytes * S);
  uint64_t* empty = full + S;
  uint64_t* mma_done = empty + S;
  uint64_t* drain = mma_done + S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(tmem_slot + 2);   // 6 floats
  int* last_flag = reinterpret_cast<int*>(tmem_slot + 8);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int rb = blockIdx.x;
  const int split = blockIdx.y;
  const int chunks = static_cast<int>(p.K / kQChunk);
  const int kc0 = split * p.chunks_per_split;
  const int kc1 = min(kc0 + p.chunks_per_split, chunks);
  const int n = kc1 - kc0;
  const bool lr = p.has_lr != 0;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), kQComputeWarps);
      mbar_init(smem_u32(&mma_done[s]), 1);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (lr && warp == kQMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 32);
    tmem_relinquish();
  }
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
  if (rb == 0 && split == 0 && tid == 0) *p.t_out = t;
  const uint32_t tmem = lr ? *tmem_slot : 0u;

  if (warp == kQProducerWarp) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_x);
      if (lr) tma_prefetch_desc(&tm_l1);
      int issued = 0;
      for (int i = 0; i < n; ++i) {
        const int s = i % S;
        if (i >= S) {
          const uint32_t ph = ((i / S) - 1) & 1;   // the fill of chunk i - S
          if (!mbar_wait(smem_u32(&empty[s]), ph, abort_flag, p.status)) break;
          if (lr && !mbar_wait(smem_u32(&mma_done[s]), ph, abort_flag, p.status)) break;
        }
        const uint32_t bar = smem_u32(&full[s]);
        uint8_t* dst = smem + s * Tile::kStageBytes;
        const int kx = (kc0 + i) * kQChunk;
        const uint32_t inv_bytes = p.inv_s != nullptr ? kQChunk * 4 : 0;
        if constexpr (sizeof(SrcT) == 2) {
          mbar_arrive_expect_tx(bar, Tile::kBytes + (lr ? Tile::kL1Bytes : 0) + inv_bytes);
          tma_load_2d(smem_u32(dst), &tm_x, bar, kx, rb * kQRows);
          if (lr) tma_load_2d(smem_u32(dst + Tile::kL1Off), &tm_l1, bar, kx, 0);
        } else {
          mbar_arrive_expect_tx(bar, Tile::kBytes + inv_bytes);
          tma_load_2d(smem_u32(dst), &tm_x, bar, kx, rb * kQRows);
          tma_load_2d(smem_u32(dst + kQRows * 128), &tm_x, bar, kx + 32, rb * kQRows);
        }
        if (inv_bytes) bulk_load(smem_u32(dst + Tile::kInvSOff), p.inv_s + kx, inv_bytes, bar);
        ++issued;
      }
      // every fill issued must land before the shared memory is released
      for (int j = max(0, issued - S); j < issued; ++j) mbar_wait_drain(smem_u32(&full[j % S]), (j / S) & 1);
    }
  } else if (warp == kQMmaWarp) {
    // ------------------------------------------------------- U = X L1 MMAs
    if (lr && lane == 0) {
      for (int i = 0; i < n; ++i) {
        const int s = i % S;
        if (!mbar_wait(smem_u32(&full[s]), (i / S) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + s * Tile::kStageBytes);
        const uint32_t b_base = a_base + Tile::kL1Off;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t ad = smem_desc(a_base + 32 * k, 16, 1024, kSwizzle128B);
          const uint64_t bd = smem_desc(b_base + 32 * k, 16, 1024, kSwizzle128B);
          mma_bf16(tmem, ad, bd, idesc_bf16(128, 32), (i > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(smem_u32(&mma_done[s]));
      }
      // all MMAs of this thread complete before TMEM is read or released
      tc_commit(smem_u32(drain));
      mbar_wait_drain(smem_u32(drain), 0);
    }
  } else {
    // ------------------------------------------------------- quantise rows
    const int row_in_tile = tid;  // compute warps are warps 0..3
    const int64_t row = static_cast<int64_t>(rb) * kQRows + row_in_tile;
    const bool row_ok = row < p.M;
    const int64_t kbytes = p.K / 2;
    for (int i = 0; i < n; ++i) {
      const int s = i % S;
      if (!mbar_wait(smem_u32(&full[s]), (i / S) & 1, abort_flag, p.status)) break;
      const uint8_t* tile = smem + s * Tile::kStageBytes;
      const int kc = kc0 + i;
      const int k0 = kc * kQChunk;

      float x[64];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float v[8];
        load8<SrcT>(tile, row_in_tile, c, v);
#pragma unroll
        for (int j = 0; j < 8; ++j) x[8 * c + j] = v[j];
      }
      if (p.inv_s != nullptr) {
        const float4* inv = reinterpret_cast<const float4*>(tile + Tile::kInvSOff);
#pragma unroll
        for (int j = 0; j < 64; j += 4) {
          const float4 sv = inv[j / 4];
          x[j] = __fmul_rn(x[j], sv.x);
          x[j + 1] = __fmul_rn(x[j + 1], sv.y);
          x[j + 2] = __fmul_rn(x[j + 2], sv.z);
          x[j + 3] = __fmul_rn(x[j + 3], sv.w);
        }
      }
      // four 16-element blocks: maxima first (this consumes every value read
      // from the stage), then release the stage: the shared-memory reads are
      // ordered before the refill's TMA writes by the proxy fence and the
      // barrier's release/acquire.
      float bmx[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        float bm = 0.0f;
#pragma unroll
        for (int j = 0; j < 16; ++j) bm = fmaxf(bm, fabsf(x[16 * b + j]));
        bmx[b] = bm;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
      uint32_t sf_word = 0;
      uint32_t codes[8];
#pragma unroll
      for (int b = 0; b < 4; b += 2) {
        const float bm0 = bmx[b], bm1 = bmx[b + 1];
        const float s0 = __fdiv_rn(__fmul_rn(bm0, rt), 6.0f);
        const float s1 = __fdiv_rn(__fmul_rn(bm1, rt), 6.0f);
        const uint32_t e2 = cvt_e4m3x2(s1, s0);  // byte 0 = block b, byte 1 = block b+1
        sf_word |= e2 << (8 * b);
        const float2 sd = e4m3x2_to_f32(e2);     // .x = block b+1, .y = block b
        const float sdb[2] = {sd.y, sd.x};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int blk = b + h;
          if (sdb[h] > 0.0f) {
            const float rq = __frcp_rn(__fmul_rn(sdb[h], t));
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              float v[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) v[j] = __fmul_rn(x[16 * blk + 8 * q + j], rq);
              codes[2 * blk + q] = cvt_e2m1x8(v);
            }
          } else {
            codes[2 * blk] = 0u;
            codes[2 * blk + 1] = 0u;
          }
        }
      }
      if (row_ok) {
        uint4* dst = reinterpret_cast<uint4*>(p.q + row * kbytes + static_cast<int64_t>(kc) * 32);
        dst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
        dst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
      }
      {
        const int64_t atom = static_cast<int64_t>(rb) * chunks + kc;
        uint32_t* sfw = reinterpret_cast<uint32_t*>(p.sf + atom * 512 + (row_in_tile & 31) * 16 +
                                                    (row_in_tile >> 5) * 4);
        *sfw = sf_word;
      }
    }
  }

  // Every role has finished (or given up); in-flight copies and MMAs drained.
  tc_fence_before();
  __syncthreads();
  const bool aborted = *abort_flag != 0;
  if (!lr || aborted) {
    if (lr && warp == kQMmaWarp) {
      tc_fence_after();
      tmem_dealloc(tmem, 32);
    }
    return;
  }

  // U partial of this K slice (TMEM lane = row): compute warps read it out.
  const int row_in_tile = tid;
  const int64_t rows_pad = static_cast<int64_t>(gridDim.x) * kQRows;
  const int64_t prow = static_cast<int64_t>(rb) * kQRows + row_in_tile;
  if (warp < kQComputeWarps) {
    tc_fence_after();
    uint32_t u[32];
    tmem_ld_32cols(tmem + (static_cast<uint32_t>(warp * 32) << 16), u);
    tmem_ld_wait();
    if (n == 0) {
#pragma unroll
      for (int j = 0; j < 32; ++j) u[j] = 0u;
    }
    float4* dst = reinterpret_cast<float4*>(p.u_part + (static_cast<int64_t>(split) * rows_pad + prow) * 32);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      dst[j] = make_float4(__uint_as_float(u[4 * j]), __uint_as_float(u[4 * j + 1]),
                           __uint_as_float(u[4 * j + 2]), __uint_as_float(u[4 * j + 3]));
    __threadfence();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kQMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 32);
  }
  if (tid == 0) {
    const int ticket = atomicAdd(&p.tickets[rb], 1);
    *last_flag = (ticket == p.splits - 1) ? 1 : 0;
  }
  __syncthreads();
  if (*last_flag && warp < kQComputeWarps) {
    // the last K slice of this row block sums the partials in slice order
    __threadfence();
    const int64_t row = static_cast<int64_t>(rb) * kQRows + row_in_tile;
    float acc[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) acc[j] = 0.0f;
    for (int sp0 = 0; sp0 < p.splits; sp0 += 2) {
      // the loads of two slices are in flight together; the sums still run
      // in slice order
      float4 w[2][8];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        if (sp0 + q < p.splits) {
          const float4* src =
              reinterpret_cast<const float4*>(p.u_part + (static_cast<int64_t>(sp0 + q) * rows_pad + prow) * 32);
#pragma unroll
          for (int j = 0; j < 8; ++j) w[q][j] = __ldcg(src + j);
        }
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        if (sp0 + q < p.splits) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            acc[4 * j] = __fadd_rn(acc[4 * j], w[q][j].x);
            acc[4 * j + 1] = __fadd_rn(acc[4 * j + 1], w[q][j].y);
            acc[4 * j + 2] = __fadd_rn(acc[4 * j + 2], w[q][j].z);
            acc[4 * j + 3] = __fadd_rn(acc[4 * j + 3], w[q][j].w);
          }
        }
      }
    }
    if (row < p.M) {
      const float ra = __frcp_rn(__fmul_rn(t, __ldg(p.t_w)));
      uint32_t hi[16], lo[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float a0 = __fmul_rn(acc[j], ra), a1 = __fmul_rn(acc[j + 1], ra);
        const uint32_t h = pack_bf16x2(a0, a1);
        hi[j / 2] = h;
        lo[j / 2] = pack_bf16x2(__fsub_rn(a0, bf16_lo(h)), __fsub_rn(a1, bf16_hi(h)));
      }
      uint4* dst2 = reinterpret_cast<uint4*>(p.u_out + row * 64);
#pragma unroll
      for (int j = 0; j < 4; ++j) dst2[j] = make_uint4(hi[4 * j], hi[4 * j + 1], hi[4 * j + 2], hi[4 * j + 3]);
#pragma unroll
      for (int j = 0; j < 4; ++j) dst2[4 + j] = make_uint4(lo[4 * j], lo[4 * j + 1], lo[4 * j + 2], lo[4 * j + 3]);
    }
  }
}

}  // namespace w4a4
