// w4a4_api.cu -- the extern "C" entry points declared in include/w4a4.h.
//
// Host code only validates arguments, encodes TMA tensor maps, sizes grids
// and enqueues the kernels of quant.cuh / gemm.cuh on the caller's stream.
// It never allocates device memory and never synchronises (except
// w4a4_device_status, which documents that it does).
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/w4a4.h"
#include "gemm.cuh"
#include "gemm2.cuh"

#include "quant.cuh"
#include "attention.cuh"
#include "mma_rate.cuh"

namespace w4a4 {

// Sticky device status word (W4A4_OK or a device-side error code).
__device__ int g_status = 0;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  bool ok = false;
  int num_sms = 0;
  int* status_ptr = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// The main pair configuration: 256 x 256 tiles, six 32 KB A/B stages, a
// three-slot scale ring, one epilogue staging buffer per warp, no alignment
// slack (the kernel checks that the dynamic shared memory base is 1024-byte
// aligned and reports W4A4_ERR_DEVICE_LAYOUT otherwise): 226 KB.
using PairMain = Gemm2Cfg<256, 6, 3, 1, false>;
// the same configuration whose epilogue can quantise for the next layer
using PairQNext = Gemm2Cfg<256, 6, 3, 1, false, true>;
// ... and the one whose epilogue can apply the rotary embedding
using PairRope = Gemm2Cfg<256, 6, 3, 1, false, false, true>;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
size_t round256(size_t v) { return (v + 255) & ~size_t(255); }

// Per-device set-up: architecture check, SM count, kernel attributes, the
// device address of the status word.  Returns W4A4_OK or an error.
int device_setup(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return W4A4_ERR_ARCH; }
  if (dev < 0 || dev >= kMaxDevices) return W4A4_ERR_ARCH;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.ready) { *out = &d; return d.ok ? W4A4_OK : W4A4_ERR_ARCH; }
  d.ready = true;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10) {
    cudaGetLastError();
    return W4A4_ERR_ARCH;
  }
  cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&d.status_ptr), g_status) != cudaSuccess) {
    cudaGetLastError();
    return W4A4_ERR_CUDA;
  }
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr) {
      cudaGetLastError();
      return W4A4_ERR_CUDA;
    }
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  bool attr_ok = true;
  attr_ok &= cudaFuncSetAttribute(quant_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  QuantTile<__nv_bfloat16>::kSmem) == cudaSuccess;
  attr_ok &= cudaFuncSetAttribute(quant_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  QuantTile<float>::kSmem) == cudaSuccess;
  attr_ok &= cudaFuncSetAttribute(quant_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  FusedQuantSmem::kBytes) == cudaSuccess;
  attr_ok &= cudaFuncSetAttribute(attn_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AttnSmem::kBytes) ==
             cudaSuccess;
  attr_ok &= cudaFuncSetAttribute(fp4_mma_rate_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kRateSmem) == cudaSuccess;
  attr_ok &= cudaFuncSetAttribute(fp4_mma_rate_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kRateSmem) == cudaSuccess;
  using G256 = GemmCfg<256, 4>;
  using G192 = GemmCfg<192, 4>;

  attr_ok &= cudaFuncSetAttribute(gemm_kernel<G256>, cudaFuncAttributeMaxDynamicSharedMemorySize, G256::SMEM) ==
             cudaSuccess;
  attr_ok &= cudaFuncSetAttribute(gemm_kernel<G192>, cudaFuncAttributeMaxDynamicSharedMemorySize, G192::SMEM) ==
             cudaSuccess;
  using P256 = PairMain;
  using P192 = Gemm2Cfg<192, 5>;
  using P64 = Gemm2Cfg<64, 6>;
  attr_ok &= cudaFuncSetAttribute(gemm2_kernel<P64>, cudaFuncAttributeMaxDynamicSharedMemorySize, P64::SMEM) ==
             cudaSuccess;
  attr_ok &= cudaFuncSetAttribute(gemm2_kernel<P256>, cudaFuncAttributeMaxDynamicSharedMemorySize, P256::SMEM) ==
             cudaSuccess;
  attr_ok &= cudaFuncSetAttribute(gemm2_kernel<P192>, cudaFuncAttributeMaxDynamicSharedMemorySize, P192::SMEM) ==
             cudaSuccess;
  attr_ok &= cudaFuncSetAttribute(gemm2_kernel<PairQNext>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  PairQNext::SMEM) == cudaSuccess;
  attr_ok &= cudaFuncSetAttribute(gemm2_kernel<PairRope>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  PairRope::SMEM) == cudaSuccess;

  if (!attr_ok) { cudaGetLastError(); return W4A4_ERR_CUDA; }
  d.ok = true;
  *out = &d;
  return W4A4_OK;
}

bool encode_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* ptr, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return g_encode(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Scale atoms viewed as u32 [row_blocks][K/64][128]; box (128, 4, rb_box).
bool encode_sf(CUtensorMap* m, const void* ptr, int64_t rows, int64_t K, uint32_t rb_box) {
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(K / 64), static_cast<cuuint64_t>(ceil_div(rows, 128))};
  const cuuint64_t strides[2] = {512, static_cast<cuuint64_t>(K / 64) * 512};
  const cuuint32_t box[3] = {128, 4, rb_box};
  const cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct QuantPlan {
  int64_t row_blocks = 0;
  int64_t grid = 0;  // CTAs of the streaming pass
  int chunks = 0, splits = 0, chunks_per_split = 0;
  int upart_slices = 0;  // K slices the low-rank partial buffer holds
  size_t off_partials = 0, off_tickets = 0, off_barrier = 0, off_upart = 0, bytes = 0;
};

// SM count the work split and the workspace size assume (B200); on another
// count the kernels stay correct, only the balance changes.
constexpr int kPlanSms = 148;

// Workspace layout (byte offsets; documented in include/w4a4.h).
constexpr size_t kWsBarrierOff = sizeof(float) * kAmaxMaxBlocks;                   // 4096
constexpr size_t kWsTicketsOff = kWsBarrierOff + 1024;                              // 160 words on 128-byte lines
constexpr int64_t kMaxTicketRowBlocks = W4A4_MAX_LOWRANK_ROWS / kQRows;             // 32768
constexpr size_t kWsUpartOff = kWsTicketsOff + sizeof(unsigned) * kMaxTicketRowBlocks;
static_assert(sizeof(unsigned) * kBarWords <= 1024, "barrier words fit their slot");
static_assert(kWsBarrierOff == W4A4_WS_BARRIER_OFFSET && kWsTicketsOff == W4A4_WS_TICKETS_OFFSET &&
                  kWsUpartOff == W4A4_WS_UPART_OFFSET,
              "layout constants of the header");

// K-slice count of the single-pass path (its tile set is co-resident: one CTA
// per (row block, slice), at most kFusedMaxChunks chunks each).
int fused_splits(int64_t row_blocks, int chunks, int64_t sms) {
  int64_t want = ceil_div(chunks, kFusedMaxChunks);
  // more slices spread the load over more SMs, but every slice adds a
  // partial U that each row's sum waits for: at most kFusedSlicesForSpread
  // slices beyond what the shared-memory budget needs
  int64_t more = row_blocks > 0 ? sms / row_blocks : 1;
  if (more > kFusedSlicesForSpread) more = kFusedSlicesForSpread;
  if (more > want) want = more;
  if (want > chunks) want = chunks;
  if (want < 1) want = 1;
  const int cps = static_cast<int>(ceil_div(chunks, want));
  return static_cast<int>(ceil_div(chunks, cps));
}

QuantPlan quant_plan(int64_t M, int64_t K, int r) {
  QuantPlan q;
  q.row_blocks = ceil_div(M, kQRows);
  q.chunks = static_cast<int>(K / kQChunk);
  // Streaming pass: CTA b of G takes chunks [b T / G, (b + 1) T / G) of the
  // (row block, chunk) sequence (T chunks in all).  With G = row_blocks x
  // splits every CTA gets one K slice of one row block; with G = kPlanSms
  // the ranges are as even as they can be and cross row blocks.  Aligned
  // slices: pick the slice count whose busiest CTA streams the fewest chunks,
  // charging four chunks per slice for the partial U it adds to a row
  // block's sum (ties: fewer slices); even ranges when the aligned plan
  // would leave SMs idle by more than that charge.
  const int64_t total = q.row_blocks * q.chunks;
  int splits = 1;
  if (total == 0) {  // an empty problem: only the fixed part of the layout
    q.grid = 0;
    q.splits = 1;
    q.chunks_per_split = q.chunks;
    q.off_partials = 0;
    q.off_barrier = kWsBarrierOff;
    q.off_tickets = kWsTicketsOff;
    q.off_upart = kWsUpartOff;
    q.upart_slices = 1;
    q.bytes = q.off_upart;
    return q;
  }
  int64_t best = -1;
  for (int sp = 1; sp <= kQMaxSplits && sp <= q.chunks; ++sp) {
    const int cps = static_cast<int>(ceil_div(q.chunks, sp));
    const int spl = static_cast<int>(ceil_div(q.chunks, cps));
    if (spl != sp) continue;
    const int64_t busiest = ceil_div(q.row_blocks * spl, kPlanSms) * cps + 4 * spl;
    if (best < 0 || busiest < best) {
      best = busiest;
      splits = spl;
    }
  }
  const int64_t even_grid = std::min<int64_t>(total, kPlanSms);
  const int64_t even_busiest = ceil_div(total, even_grid) + 4 * (ceil_div(even_grid, q.row_blocks) + 1);
  // (measured: even ranges gain on 16896 x 24576, 8 %, and lose 2 % where
  // they win by less than a few percent on paper, e.g. 16896 x 6144)
  const bool aligned = q.row_blocks * splits <= kPlanSms && best <= even_busiest + even_busiest / 32;
  q.grid = aligned ? q.row_blocks * splits : even_grid;
  // partial U per row block: one per CTA whose range touches it
  q.splits = static_cast<int>(std::min<int64_t>(q.chunks, aligned ? splits : ceil_div(q.grid, q.row_blocks) + 1));
  q.chunks_per_split = q.chunks;
  // the single-pass path has its own K slices (only when its tile set fits
  // on the device at once: the condition launch_quant_fused checks)
  int fused = 1;
  if (q.row_blocks <= kPlanSms) {
    const int sp = fused_splits(q.row_blocks, q.chunks, kPlanSms);
    if (ceil_div(q.chunks, sp) <= kFusedMaxChunks && q.row_blocks * sp <= kPlanSms) fused = sp;
  }
  const int slices_max = std::max(q.splits, fused);
  // Fixed layout, the same for every M, K and r (so that one workspace
  // serves any sequence of calls): amax partial maxima; the single-pass
  // grid barrier (launch generation, counters and maximum words per
  // generation parity); one low-rank ticket per 128-row block up to
  // kMaxTicketRowBlocks (zero at rest: each kernel clears the ones it used);
  // then the fp32 low-rank partial sums, whose size alone depends on M.
  q.off_partials = 0;
  q.off_barrier = kWsBarrierOff;
  q.off_tickets = kWsTicketsOff;
  q.off_upart = kWsUpartOff;
  q.upart_slices = slices_max;
  const size_t upart = r > 0 ? sizeof(float) * static_cast<size_t>(slices_max) * q.row_blocks * kQRows * 32 : 0;
  q.bytes = q.off_upart + round256(upart);
  return q;
}

// Largest K: the tensor-amax pass gives every CTA kAmaxThreads 16-byte
// column segments of a row and keeps at most kAmaxMaxBlocks partial maxima,
// so a row spans at most kAmaxMaxBlocks x kAmaxThreads segments: 2^20 fp32
// (weight) or 2^21 bf16 columns.  One bound for every entry point.
constexpr int64_t kMaxK = int64_t(kAmaxMaxBlocks) * kAmaxThreads * 4;
static_assert(kMaxK == (int64_t(1) << 20) && kMaxK == W4A4_MAX_K, "K bound of the header");
// Largest column count of fp8_quantize (bf16 only: eight per segment).
constexpr int64_t kFp8MaxCols = int64_t(kAmaxMaxBlocks) * kAmaxThreads * 8;

bool valid_k(int64_t K) { return K >= 64 && K % 64 == 0 && K <= kMaxK; }

// Rows the per-row-block low-rank counters of a workspace cover.
bool valid_lowrank_rows(int64_t M, int r) { return r == 0 || M <= W4A4_MAX_LOWRANK_ROWS; }

// Single-pass activation quantisation: every (row block, K slice) tile must
// be resident at once, one CTA per SM.  Returns W4A4_OK, or -1 when the shape
// or the device does not allow it (the caller then runs the two-pass path).
int launch_quant_fused(const __nv_bfloat16* X, int64_t M, int64_t K, int64_t ld, const float* inv_s,
                       const void* L1t, int r, const float* t_w, uint8_t* q, uint8_t* sf, float* t_out, void* U,
                       void* ws, cudaStream_t stream, DeviceInfo* dev) {
  const QuantPlan plan = quant_plan(M, K, r);
  const int64_t rb = plan.row_blocks;
  const int chunks = plan.chunks;
  if (rb < 1 || rb > dev->num_sms) return -1;
  const int splits = fused_splits(rb, chunks, dev->num_sms);
  const int cps = static_cast<int>(ceil_div(chunks, splits));
  if (cps > kFusedMaxChunks || rb * splits > dev->num_sms || splits > plan.upart_slices) return -1;

  uint8_t* w = static_cast<uint8_t*>(ws);
  // one ticket per row block (zero at rest: the kernel clears them before it
  // ends) and the grid barrier's words
  unsigned* tickets = reinterpret_cast<unsigned*>(w + plan.off_tickets);
  unsigned* barrier = reinterpret_cast<unsigned*>(w + plan.off_barrier);
  CUtensorMap tm_x, tm_l1;
  if (!encode_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                 static_cast<uint64_t>(ld) * 2, 64u, 128u, CU_TENSOR_MAP_SWIZZLE_128B))
    return W4A4_ERR_CUDA;
  if (r > 0) {
    if (!encode_2d(&tm_l1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L1t, static_cast<uint64_t>(K), static_cast<uint64_t>(r),
                   static_cast<uint64_t>(K) * 2, 64u, static_cast<uint32_t>(r), CU_TENSOR_MAP_SWIZZLE_128B))
      return W4A4_ERR_CUDA;
  } else {
    tm_l1 = tm_x;
  }
  // codes, written by TMA: 32 rows x 32 bytes (one 64-wide chunk) per box
  CUtensorMap tm_q;
  if (!encode_2d(&tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, static_cast<uint64_t>(K / 2), static_cast<uint64_t>(M),
                 static_cast<uint64_t>(K / 2), 32u, 32u, CU_TENSOR_MAP_SWIZZLE_NONE))
    return W4A4_ERR_CUDA;
  QuantParams p;
  p.M = M;
  p.K = K;
  p.inv_s = inv_s;
  p.partials = reinterpret_cast<float*>(w + plan.off_partials);
  p.n_partials = static_cast<int>(rb * splits);
  p.t_w = t_w;
  p.q = q;
  p.sf = sf;
  p.t_out = t_out;
  p.u_part = reinterpret_cast<float*>(w + plan.off_upart);
  p.u_out = static_cast<__nv_bfloat16*>(U);
  p.tickets = nullptr;
  p.chunks_per_split = cps;
  p.splits = splits;
  p.row_blocks = static_cast<int>(rb);
  p.has_lr = r > 0 ? 1 : 0;
  p.r = r;
  p.status = dev->status_ptr;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(rb * splits), 1, 1);
  cfg.blockDim = dim3(kFThreads, 1, 1);
  cfg.dynamicSmemBytes = FusedQuantSmem::kBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // set-up overlaps the previous kernel
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, quant_fused_kernel, tm_x, tm_l1, tm_q, p, tickets, barrier) == cudaSuccess) return W4A4_OK;
  cudaGetLastError();
  cfg.numAttrs = 1;  // without the programmatic attribute
  if (cudaLaunchKernelEx(&cfg, quant_fused_kernel, tm_x, tm_l1, tm_q, p, tickets, barrier) == cudaSuccess) return W4A4_OK;
  cudaGetLastError();
  return -1;  // not co-resident on this device: fall back
}

template <typename SrcT>
int launch_quant(const SrcT* X, int64_t M, int64_t K, int64_t ld, const float* inv_s, const void* L1t, int r,
                 const float* t_w, uint8_t* q, uint8_t* sf, float* t_out, void* U, void* ws,
                 cudaStream_t stream, DeviceInfo* dev, const float* amax_in = nullptr) {
  // With the tensor amax given (by the producer of X), the quantise pass
  // alone streams X once at any size.
  if constexpr (sizeof(SrcT) == 2) {
    if (amax_in == nullptr) {
      const int st = launch_quant_fused(X, M, K, ld, inv_s, L1t, r, t_w, q, sf, t_out, U, ws, stream, dev);
      if (st != -1) return st;
    }
  }
  const QuantPlan plan = quant_plan(M, K, r);
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* partials = reinterpret_cast<float*>(w + plan.off_partials);
  int* tickets = reinterpret_cast<int*>(w + plan.off_tickets);
  float* upart = reinterpret_cast<float*>(w + plan.off_upart);

  // pass 1: column-segment CTAs (x) times row bands (y), about four CTAs per
  // SM, at most kAmaxMaxBlocks partial maxima
  constexpr int EPV = 16 / sizeof(SrcT);
  const int64_t gx = ceil_div(K / EPV, kAmaxThreads);
  int64_t gy = ceil_div(4 * static_cast<int64_t>(dev->num_sms), gx);
  if (gy > kAmaxMaxBlocks / gx) gy = kAmaxMaxBlocks / gx;
  if (gy > M) gy = M;
  if (gy < 1) gy = 1;
  const int64_t rows_per = ceil_div(M, gy);
  gy = ceil_div(M, rows_per);
  const int64_t grid1 = gx * gy;
  if (amax_in == nullptr) {
    amax_kernel<SrcT><<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)), kAmaxThreads, 0, stream>>>(
        X, M, K, ld, inv_s, partials, static_cast<int>(rows_per));
    if (cudaGetLastError() != cudaSuccess) return W4A4_ERR_CUDA;
  }

  CUtensorMap tm_x, tm_l1;
  const bool is_bf16 = sizeof(SrcT) == 2;
  if (!encode_2d(&tm_x, is_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, X,
                 static_cast<uint64_t>(K), static_cast<uint64_t>(M), static_cast<uint64_t>(ld) * sizeof(SrcT),
                 is_bf16 ? 64u : 32u, 128u, CU_TENSOR_MAP_SWIZZLE_128B))
    return W4A4_ERR_CUDA;
  if (r > 0) {
    if (!encode_2d(&tm_l1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L1t, static_cast<uint64_t>(K), static_cast<uint64_t>(r),
                   static_cast<uint64_t>(K) * 2, 64u, static_cast<uint32_t>(r), CU_TENSOR_MAP_SWIZZLE_128B))
      return W4A4_ERR_CUDA;
  } else {
    tm_l1 = tm_x;  // unused
  }
  // codes, written by TMA: 32 rows x 32 bytes (one 64-wide chunk) per box
  CUtensorMap tm_q;
  if (!encode_2d(&tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, static_cast<uint64_t>(K / 2), static_cast<uint64_t>(M),
                 static_cast<uint64_t>(K / 2), 32u, 32u, CU_TENSOR_MAP_SWIZZLE_NONE))
    return W4A4_ERR_CUDA;
  QuantParams p;
  p.M = M;
  p.K = K;
  p.inv_s = inv_s;
  p.partials = amax_in != nullptr ? amax_in : partials;
  p.n_partials = amax_in != nullptr ? 1 : static_cast<int>(grid1);
  p.t_w = t_w;
  p.q = q;
  p.sf = sf;
  p.t_out = t_out;
  p.u_part = upart;
  p.u_out = static_cast<__nv_bfloat16*>(U);
  p.tickets = tickets;
  p.chunks_per_split = plan.chunks;  // (the streaming kernel takes equal ranges, not K slices)
  p.splits = 1;
  p.row_blocks = static_cast<int>(plan.row_blocks);
  p.has_lr = r > 0 ? 1 : 0;
  p.r = r;
  p.status = dev->status_ptr;
  // one CTA per SM at most, each taking its share of the (row block, chunk)
  // sequence (the plan's grid, or fewer CTAs on a smaller device: then each
  // row block is touched by no more pieces than the workspace holds)
  const int64_t grid2 = std::min<int64_t>(plan.grid, dev->num_sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid2), 1, 1);
  cfg.blockDim = dim3(kQThreads, 1, 1);
  cfg.dynamicSmemBytes = QuantTile<SrcT>::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // set-up overlaps the previous kernel
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, quant_kernel<SrcT>, tm_x, tm_l1, tm_q, p) != cudaSuccess) {
    cudaGetLastError();
    return W4A4_ERR_CUDA;
  }
  return W4A4_OK;
}

template <class C>
int launch_gemm_cfg(const uint8_t* Xq, const uint8_t* Xsf, const float* t_x, const void* U, int64_t M, int64_t N,
                    int64_t K, const uint8_t* Wq, const uint8_t* Wsf, const float* t_w, const void* L2t, int r,
                    const void* bias, int epi, void* Y, int64_t ldy, const float* next_inv_s, unsigned* next_amax,
                    cudaStream_t stream, DeviceInfo* dev) {
  CUtensorMap ta, tb, tsa, tsb, tu, tl;
  if (!encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, Xq, static_cast<uint64_t>(K / 2), static_cast<uint64_t>(M),
                 static_cast<uint64_t>(K / 2), 128u, 128u, CU_TENSOR_MAP_SWIZZLE_128B))
    return W4A4_ERR_CUDA;
  if (!encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, static_cast<uint64_t>(K / 2), static_cast<uint64_t>(N),
                 static_cast<uint64_t>(K / 2), 128u, static_cast<uint32_t>(C::BN), CU_TENSOR_MAP_SWIZZLE_128B))
    return W4A4_ERR_CUDA;
  if (!encode_sf(&tsa, Xsf, M, K, 1)) return W4A4_ERR_CUDA;
  if (!encode_sf(&tsb, Wsf, N, K, 2)) return W4A4_ERR_CUDA;
  if (r > 0) {
    // U = [hi | lo], rows of 2r bf16; L2t rows of r bf16 (swizzle = row width)
    if (!encode_2d(&tu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, U, static_cast<uint64_t>(2 * r), static_cast<uint64_t>(M),
                   static_cast<uint64_t>(4 * r), static_cast<uint32_t>(2 * r), 128u,
                   r == 32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
      return W4A4_ERR_CUDA;
    if (!encode_2d(&tl, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L2t, static_cast<uint64_t>(r), static_cast<uint64_t>(N),
                   static_cast<uint64_t>(2 * r), static_cast<uint32_t>(r), static_cast<uint32_t>(C::BN),
                   r == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B))
      return W4A4_ERR_CUDA;
  } else {
    tu = ta;
    tl = ta;
  }
  GemmParams p;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.ldy = ldy;
  p.t_x = t_x;
  p.t_w = t_w;
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.Y = static_cast<__nv_bfloat16*>(Y);
  p.has_lr = r > 0 ? 1 : 0;
  p.r = r;
  p.epi = epi;
  p.status = dev->status_ptr;
  p.next_inv_s = next_inv_s;
  p.next_amax = next_amax;
  p.n_plain = static_cast<int>(N);
  p.H = nullptr;
  p.ldh = 0;
  p.q_next = nullptr;
  p.sf_next = nullptr;
  p.t_next = nullptr;
  p.ldq = 0;
  p.next_K = 0;
  p.q_col0 = 0;
  p.n_rope = 0;
  p.d_head = 0;
  p.rope = nullptr;
  p.ld_rope = 0;
  const int64_t tiles = ceil_div(M, C::BM) * ceil_div(N, C::BN);
  const int64_t grid = tiles < dev->num_sms ? tiles : dev->num_sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // set-up overlaps the previous kernel
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, gemm_kernel<C>, ta, tb, tsa, tsb, tu, tl, p) != cudaSuccess) {
    cudaGetLastError();
    return W4A4_ERR_CUDA;
  }
  return W4A4_OK;
}

// Quantise-into-epilogue outputs of the CTA-pair kernel (q == nullptr: off).
struct QuantNext {
  uint8_t* q = nullptr;
  uint8_t* sf = nullptr;
  const float* t = nullptr;
  int64_t ldq = 0, K = 0, col = 0;
};

// Rotary embedding of the leading plain outputs (n_rope == 0: off).
struct RopeArgs {
  int64_t n_rope = 0, d_head = 0, ld = 0;
  const float* table = nullptr;
};

// The CTA-pair kernels: 256 x BN tiles on two SMs (cluster of 2).
template <class C>
int launch_gemm_pair(const uint8_t* Xq, const uint8_t* Xsf, const float* t_x, const void* U, int64_t M, int64_t N,
                     int64_t K, const uint8_t* Wq, const uint8_t* Wsf, const float* t_w, const void* L2t, int r,
                     const void* bias, int epi, void* Y, int64_t ldy, const float* next_inv_s, unsigned* next_amax,
                     cudaStream_t stream, DeviceInfo* dev, int64_t n_plain = -1, void* H = nullptr,
                     int64_t ldh = 0, QuantNext qn = QuantNext(), RopeArgs ra = RopeArgs()) {
  if (n_plain < 0) n_plain = N;
  if (ra.n_rope > 0 && !C::ROPE) return W4A4_ERR_ARG;
  // SwiGLU outputs fill 32-column boxes from two 32-column accumulator blocks
  if (n_plain < N && (C::BN % 64 != 0 || n_plain % C::BN != 0)) return W4A4_ERR_SHAPE;
  CUtensorMap ta, tb, tsa, tsb, tu, tl, ty, th;
  if (!encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, Xq, static_cast<uint64_t>(K / 2), static_cast<uint64_t>(M),
                 static_cast<uint64_t>(K / 2), 128u, 128u, CU_TENSOR_MAP_SWIZZLE_128B))
    return W4A4_ERR_CUDA;
  if (!encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, static_cast<uint64_t>(K / 2), static_cast<uint64_t>(N),
                 static_cast<uint64_t>(K / 2), 128u, static_cast<uint32_t>(C::BH), CU_TENSOR_MAP_SWIZZLE_128B))
    return W4A4_ERR_CUDA;
  if (!encode_sf(&tsa, Xsf, M, K, 1)) return W4A4_ERR_CUDA;
  if (!encode_sf(&tsb, Wsf, N, K, static_cast<uint32_t>(C::SFB_RB))) return W4A4_ERR_CUDA;
  // plain outputs Y [M, n_plain] and SwiGLU outputs H [M, (N - n_plain) / 2],
  // both written in 32 x 32 boxes
  if (n_plain > 0 && Y != nullptr && !encode_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, static_cast<uint64_t>(n_plain),
                                static_cast<uint64_t>(M), static_cast<uint64_t>(ldy) * 2, 32u, 32u,
                                CU_TENSOR_MAP_SWIZZLE_64B))
    return W4A4_ERR_CUDA;
  if (n_plain < N && H != nullptr) {
    if (!encode_2d(&th, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, H, static_cast<uint64_t>((N - n_plain) / 2),
                   static_cast<uint64_t>(M), static_cast<uint64_t>(ldh) * 2, 32u, 32u, CU_TENSOR_MAP_SWIZZLE_64B))
      return W4A4_ERR_CUDA;
    if (n_plain == 0 || Y == nullptr) ty = th;  // unused
  } else if (n_plain > 0 && Y != nullptr) {
    th = ty;  // unused
  } else {
    // neither bf16 output is stored (quantised outputs only): the maps are
    // never used; give them a valid encoding
    if (!encode_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_UINT8, Xq, static_cast<uint64_t>(K / 2), static_cast<uint64_t>(M),
                   static_cast<uint64_t>(K / 2), 32u, 32u, CU_TENSOR_MAP_SWIZZLE_NONE))
      return W4A4_ERR_CUDA;
    th = ty;
  }
  if (r > 0) {
    // U = [hi | lo], rows of 2r bf16; L2t rows of r bf16 (swizzle = row width)
    if (!encode_2d(&tu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, U, static_cast<uint64_t>(2 * r), static_cast<uint64_t>(M),
                   static_cast<uint64_t>(4 * r), static_cast<uint32_t>(2 * r), 128u,
                   r == 32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
      return W4A4_ERR_CUDA;
    if (!encode_2d(&tl, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L2t, static_cast<uint64_t>(r), static_cast<uint64_t>(N),
                   static_cast<uint64_t>(2 * r), static_cast<uint32_t>(r), static_cast<uint32_t>(C::BH),
                   r == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B))
      return W4A4_ERR_CUDA;
  } else {
    tu = ta;
    tl = ta;
  }
  GemmParams p;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.ldy = ldy;
  p.t_x = t_x;
  p.t_w = t_w;
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.Y = static_cast<__nv_bfloat16*>(Y);
  p.has_lr = r > 0 ? 1 : 0;
  p.r = r;
  p.epi = epi;
  p.status = dev->status_ptr;
  p.next_inv_s = next_inv_s;
  p.next_amax = next_amax;
  p.n_plain = static_cast<int>(n_plain);
  p.H = static_cast<__nv_bfloat16*>(H);
  p.ldh = ldh;
  p.q_next = qn.q;
  p.sf_next = qn.sf;
  p.t_next = qn.t;
  p.ldq = qn.ldq;
  p.next_K = static_cast<int>(qn.K);
  p.q_col0 = static_cast<int>(qn.col);
  p.n_rope = static_cast<int>(ra.n_rope);
  p.d_head = static_cast<int>(ra.d_head);
  p.rope = ra.table;
  p.ld_rope = ra.ld;
  const int64_t tiles = ceil_div(M, 2 * C::BM) * ceil_div(N, C::BN);
  const int64_t max_pairs = dev->num_sms / 2;
  const int64_t pairs = tiles < max_pairs ? tiles : max_pairs;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // set-up overlaps the previous kernel
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, gemm2_kernel<C>, ta, tb, tsa, tsb, tu, tl, ty, th, p) != cudaSuccess) {
    cudaGetLastError();
    return W4A4_ERR_CUDA;
  }
  return W4A4_OK;
}

int check_gemm_args(const uint8_t* Xq, const uint8_t* Xsf, const float* t_x, const void* U, int64_t M, int64_t N,
                    int64_t K, const uint8_t* Wq, const uint8_t* Wsf, const float* t_w, const void* L2t, int r,
                    const void* bias, int epi, const void* Y, int64_t ldy) {
  if (M < 0 || N <= 0 || N % 8 != 0 || !valid_k(K) || M > (int64_t(1) << 30) || N > (int64_t(1) << 30))
    return W4A4_ERR_SHAPE;
  if (r != 0 && r != 16 && r != 32) return W4A4_ERR_SHAPE;
  if (epi != W4A4_EPI_NONE && epi != W4A4_EPI_GELU_TANH) return W4A4_ERR_ARG;
  if (ldy < N || ldy % 8 != 0) return W4A4_ERR_SHAPE;
  if (M == 0) return W4A4_OK;  // empty problem
  if (!Xq || !Xsf || !t_x || !Wq || !Wsf || !t_w || !Y) return W4A4_ERR_NULL;
  if (r > 0 && (!U || !L2t)) return W4A4_ERR_NULL;
  if (!aligned16(Xq) || !aligned16(Xsf) || !aligned16(Wq) || !aligned16(Wsf) || !aligned16(Y) ||
      (bias && !aligned16(bias)) || (U && !aligned16(U)) || (L2t && !aligned16(L2t)))
    return W4A4_ERR_ALIGN;
  return W4A4_OK;
}

}  // namespace
}  // namespace w4a4

using namespace w4a4;

extern "C" {

size_t nvfp4_sf_bytes(int64_t rows, int64_t K) {
  if (rows < 0 || K <= 0 || K % 64 != 0) return 0;
  return static_cast<size_t>(ceil_div(rows, 128)) * 128 * static_cast<size_t>(K / 16);
}

size_t nvfp4_quant_workspace_bytes(int64_t M, int64_t K, int r) {
  if (M < 0 || !valid_k(K) || (r != 0 && r != 16 && r != 32) || !valid_lowrank_rows(M, r)) return 0;
  return quant_plan(M, K, r).bytes;
}

size_t w4a4_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
  if (M < 0 || N <= 0 || N % 8 != 0 || !valid_k(K) || (r != 0 && r != 16 && r != 32) || !valid_lowrank_rows(M, r))
    return 0;
  size_t b = quant_plan(M, K, r).bytes;
  b += round256(static_cast<size_t>(M) * static_cast<size_t>(K / 2));  // Xq
  b += round256(nvfp4_sf_bytes(M, K));                                  // Xsf
  b += 256;                                                             // t_x
  b += round256(r > 0 ? static_cast<size_t>(M) * 64 * 2 : 0);           // U hi|lo
  return b;
}

static int quantize_act_impl(const void* X, int64_t M, int64_t K, int64_t ldx, const float* inv_s, const void* L1t,
                             int r, const float* t_w, uint8_t* Xq, uint8_t* Xsf, float* t_x, void* U, void* workspace,
                             size_t workspace_bytes, void* stream, const float* amax_in) {
  if (M < 0 || !valid_k(K) || ldx < K || ldx % 8 != 0 || M > (int64_t(1) << 30)) return W4A4_ERR_SHAPE;
  if (r != 0 && r != 16 && r != 32) return W4A4_ERR_SHAPE;
  if (!valid_lowrank_rows(M, r)) return W4A4_ERR_SHAPE;
  if (M == 0) return W4A4_OK;  // empty problem: nothing to check further, nothing enqueued
  if (!X || !Xq || !Xsf || !t_x) return W4A4_ERR_NULL;
  if (r > 0 && (!L1t || !t_w || !U)) return W4A4_ERR_NULL;
  if (!aligned16(X) || !aligned16(Xq) || !aligned16(Xsf) || (inv_s && !aligned16(inv_s)) ||
      (L1t && !aligned16(L1t)) || (U && !aligned16(U)) || (workspace && !aligned16(workspace)))
    return W4A4_ERR_ALIGN;
  if (!workspace || workspace_bytes < nvfp4_quant_workspace_bytes(M, K, r)) return W4A4_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  int st = device_setup(&dev);
  if (st != W4A4_OK) return st;
  return launch_quant<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(X), M, K, ldx, inv_s, L1t, r, t_w, Xq, Xsf,
                                     t_x, U, workspace, static_cast<cudaStream_t>(stream), dev, amax_in);
}

int nvfp4_quantize_act(const void* X, int64_t M, int64_t K, int64_t ldx, const float* inv_s, const void* L1t, int r,
                       const float* t_w, uint8_t* Xq, uint8_t* Xsf, float* t_x, void* U, void* workspace,
                       size_t workspace_bytes, void* stream) {
  return quantize_act_impl(X, M, K, ldx, inv_s, L1t, r, t_w, Xq, Xsf, t_x, U, workspace, workspace_bytes, stream,
                           nullptr);
}

int nvfp4_quantize_act_with_amax(const void* X, int64_t M, int64_t K, int64_t ldx, const float* inv_s,
                                 const void* L1t, int r, const float* t_w, const float* amax, uint8_t* Xq,
                                 uint8_t* Xsf, float* t_x, void* U, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  if (M != 0 && !amax) return W4A4_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(amax) % 4 != 0) return W4A4_ERR_ALIGN;
  return quantize_act_impl(X, M, K, ldx, inv_s, L1t, r, t_w, Xq, Xsf, t_x, U, workspace, workspace_bytes, stream,
                           amax);
}

int nvfp4_pack_weight(const void* R, int src_dtype, int64_t N, int64_t K, int64_t ldr, uint8_t* Wq, uint8_t* Wsf,
                      float* t_w, void* workspace, size_t workspace_bytes, void* stream) {
  if (src_dtype != W4A4_SRC_BF16 && src_dtype != W4A4_SRC_F32) return W4A4_ERR_ARG;
  const int64_t vec = src_dtype == W4A4_SRC_BF16 ? 8 : 4;
  if (N < 0 || !valid_k(K) || ldr < K || ldr % vec != 0 || N > (int64_t(1) << 30)) return W4A4_ERR_SHAPE;
  if (N == 0) return W4A4_OK;  // empty problem
  if (!R || !Wq || !Wsf || !t_w) return W4A4_ERR_NULL;
  if (!aligned16(R) || !aligned16(Wq) || !aligned16(Wsf) || (workspace && !aligned16(workspace)))
    return W4A4_ERR_ALIGN;
  if (!workspace || workspace_bytes < nvfp4_quant_workspace_bytes(N, K, 0)) return W4A4_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  int st = device_setup(&dev);
  if (st != W4A4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (src_dtype == W4A4_SRC_BF16)
    return launch_quant<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(R), N, K, ldr, nullptr, nullptr, 0, nullptr,
                                       Wq, Wsf, t_w, nullptr, workspace, s, dev);
  return launch_quant<float>(static_cast<const float*>(R), N, K, ldr, nullptr, nullptr, 0, nullptr, Wq, Wsf, t_w,
                             nullptr, workspace, s, dev);
}

static int gemm_dispatch(const uint8_t* Xq, const uint8_t* Xsf, const float* t_x, const void* U, int64_t M, int64_t N,
                         int64_t K, const uint8_t* Wq, const uint8_t* Wsf, const float* t_w, const void* L2t, int r,
                         const void* bias, int epilogue, void* Y, int64_t ldy, const float* next_inv_s,
                         unsigned* next_amax, void* stream) {
  int st = check_gemm_args(Xq, Xsf, t_x, U, M, N, K, Wq, Wsf, t_w, L2t, r, bias, epilogue, Y, ldy);
  if (st != W4A4_OK || M == 0) return st;
  DeviceInfo* dev = nullptr;
  st = device_setup(&dev);
  if (st != W4A4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // CTA pairs (256 x 256 tiles) once there are at least two row blocks.
  // A single row block: CTA pairs with 256 x 64 tiles (the second CTA's rows
  // are past M: TMA fills them with zeros and the store drops them) while
  // that gives at most two tiles per pair, so a small layer streams its
  // weight through many SMs; else single-CTA 128 x 192 / 128 x 256 tiles.
  if (M > 128)
    return launch_gemm_pair<PairMain>(Xq, Xsf, t_x, U, M, N, K, Wq, Wsf, t_w, L2t, r, bias, epilogue, Y, ldy,
                                              next_inv_s, next_amax, s, dev);
  if (ceil_div(N, 64) <= static_cast<int64_t>(dev->num_sms))
    return launch_gemm_pair<Gemm2Cfg<64, 6>>(Xq, Xsf, t_x, U, M, N, K, Wq, Wsf, t_w, L2t, r, bias, epilogue, Y, ldy,
                                             next_inv_s, next_amax, s, dev);
  if (N % 192 == 0)
    return launch_gemm_cfg<GemmCfg<192, 4>>(Xq, Xsf, t_x, U, M, N, K, Wq, Wsf, t_w, L2t, r, bias, epilogue, Y, ldy,
                                            next_inv_s, next_amax, s, dev);
  return launch_gemm_cfg<GemmCfg<256, 4>>(Xq, Xsf, t_x, U, M, N, K, Wq, Wsf, t_w, L2t, r, bias, epilogue, Y, ldy,
                                          next_inv_s, next_amax, s, dev);
}

int w4a4_gemm(const uint8_t* Xq, const uint8_t* Xsf, const float* t_x, const void* U, int64_t M, int64_t N, int64_t K,
              const uint8_t* Wq, const uint8_t* Wsf, const float* t_w, const void* L2t, int r, const void* bias,
              int epilogue, void* Y, int64_t ldy, void* stream) {
  return gemm_dispatch(Xq, Xsf, t_x, U, M, N, K, Wq, Wsf, t_w, L2t, r, bias, epilogue, Y, ldy, nullptr, nullptr,
                       stream);
}

int w4a4_gemm_next_amax(const uint8_t* Xq, const uint8_t* Xsf, const float* t_x, const void* U, int64_t M, int64_t N,
                        int64_t K, const uint8_t* Wq, const uint8_t* Wsf, const float* t_w, const void* L2t, int r,
                        const void* bias, int epilogue, void* Y, int64_t ldy, const float* next_inv_s,
                        float* next_amax, void* stream) {
  if (M != 0 && !next_amax) return W4A4_ERR_NULL;
  if ((next_inv_s && !aligned16(next_inv_s)) || reinterpret_cast<uintptr_t>(next_amax) % 4 != 0)
    return W4A4_ERR_ALIGN;
  return gemm_dispatch(Xq, Xsf, t_x, U, M, N, K, Wq, Wsf, t_w, L2t, r, bias, epilogue, Y, ldy, next_inv_s,
                       reinterpret_cast<unsigned*>(next_amax), stream);
}

int w4a4_gemm_swiglu(const uint8_t* Xq, const uint8_t* Xsf, const float* t_x, const void* U, int64_t M, int64_t N,
                     int64_t K, const uint8_t* Wq, const uint8_t* Wsf, const float* t_w, const void* L2t, int r,
                     const void* bias, int64_t n_plain, void* Y, int64_t ldy, void* H, int64_t ldh,
                     const float* next_inv_s, float* next_amax, void* stream) {
  if (n_plain < 0 || n_plain >= N || n_plain % 256 != 0 || (N - n_plain) % 32 != 0) return W4A4_ERR_SHAPE;
  const int64_t n_h = (N - n_plain) / 2;
  if (ldh < n_h || ldh % 8 != 0 || (n_plain > 0 && (ldy < n_plain || ldy % 8 != 0))) return W4A4_ERR_SHAPE;
  // the common checks, with the plain part's columns standing for Y's
  int st = check_gemm_args(Xq, Xsf, t_x, U, M, N, K, Wq, Wsf, t_w, L2t, r, bias, W4A4_EPI_NONE,
                           n_plain > 0 ? Y : H, N);
  if (st != W4A4_OK || M == 0) return st;
  if (!H || (n_plain > 0 && !Y)) return W4A4_ERR_NULL;
  if (!aligned16(H) || (n_plain > 0 && !aligned16(Y)) || (next_inv_s && !aligned16(next_inv_s)) ||
      reinterpret_cast<uintptr_t>(next_amax) % 4 != 0)
    return W4A4_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  st = device_setup(&dev);
  if (st != W4A4_OK) return st;
  return launch_gemm_pair<PairMain>(Xq, Xsf, t_x, U, M, N, K, Wq, Wsf, t_w, L2t, r, bias, W4A4_EPI_NONE, Y, ldy,
                                    next_inv_s, reinterpret_cast<unsigned*>(next_amax),
                                    static_cast<cudaStream_t>(stream), dev, n_plain, H, ldh);
}

int w4a4_gemm_rope(const uint8_t* Xq, const uint8_t* Xsf, const float* t_x, const void* U, int64_t M, int64_t N,
                   int64_t K, const uint8_t* Wq, const uint8_t* Wsf, const float* t_w, const void* L2t, int r,
                   const void* bias, int64_t n_rope, int64_t d_head, const float* rope, int64_t ld_rope,
                   int64_t n_plain, void* Y, int64_t ldy, void* H, int64_t ldh, const float* next_inv_s,
                   float* next_amax, void* stream) {
  if (n_plain < 0 || n_plain > N || (n_plain < N && (n_plain % 256 != 0 || (N - n_plain) % 32 != 0)))
    return W4A4_ERR_SHAPE;
  if (d_head < 32 || d_head % 32 != 0 || n_rope <= 0 || n_rope % d_head != 0 || n_rope > n_plain ||
      ld_rope < d_head || ld_rope % 4 != 0 || ld_rope > (int64_t(1) << 30))
    return W4A4_ERR_SHAPE;
  const bool swiglu = n_plain < N;
  if (swiglu && (ldh < (N - n_plain) / 2 || ldh % 8 != 0)) return W4A4_ERR_SHAPE;
  if (ldy < n_plain || ldy % 8 != 0) return W4A4_ERR_SHAPE;
  int st = check_gemm_args(Xq, Xsf, t_x, U, M, N, K, Wq, Wsf, t_w, L2t, r, bias, W4A4_EPI_NONE, Y, N);
  if (st != W4A4_OK || M == 0) return st;
  if (!rope || (swiglu && !H)) return W4A4_ERR_NULL;
  if (!aligned16(rope) || (swiglu && !aligned16(H)) || (next_inv_s && !aligned16(next_inv_s)) ||
      reinterpret_cast<uintptr_t>(next_amax) % 4 != 0)
    return W4A4_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  st = device_setup(&dev);
  if (st != W4A4_OK) return st;
  RopeArgs ra;
  ra.n_rope = n_rope;
  ra.d_head = d_head;
  ra.ld = ld_rope;
  ra.table = rope;
  return launch_gemm_pair<PairRope>(Xq, Xsf, t_x, U, M, N, K, Wq, Wsf, t_w, L2t, r, bias, W4A4_EPI_NONE, Y, ldy,
                                    next_inv_s, reinterpret_cast<unsigned*>(next_amax),
                                    static_cast<cudaStream_t>(stream), dev, n_plain, swiglu ? H : nullptr, ldh,
                                    QuantNext(), ra);
}

int w4a4_gemm_quantize_next(const uint8_t* Xq, const uint8_t* Xsf, const float* t_x, const void* U, int64_t M,
                            int64_t N, int64_t K, const uint8_t* Wq, const uint8_t* Wsf, const float* t_w,
                            const void* L2t, int r, const void* bias, int epilogue, int64_t n_plain, void* Y,
                            int64_t ldy, void* H, int64_t ldh, const float* next_inv_s, const float* next_t,
                            uint8_t* next_q, int64_t next_ldq, uint8_t* next_sf, int64_t next_K, int64_t next_col,
                            float* next_amax, void* stream) {
  if (n_plain < 0 || n_plain > N || n_plain % 256 != 0 && n_plain != N) return W4A4_ERR_SHAPE;
  const bool swiglu = n_plain < N;
  if (swiglu && ((N - n_plain) % 32 != 0 || epilogue != W4A4_EPI_NONE)) return W4A4_ERR_SHAPE;
  const int64_t n_out = swiglu ? (N - n_plain) / 2 : N;  // the outputs quantised for the next layer
  if (n_out % 32 != 0 || next_K % 64 != 0 || next_col < 0 || next_col % 64 != 0 || next_col + n_out > next_K ||
      next_ldq < next_K / 2 || next_ldq % 16 != 0 || next_K > kMaxK)
    return W4A4_ERR_SHAPE;
  if (swiglu && H != nullptr && (ldh < n_out || ldh % 8 != 0)) return W4A4_ERR_SHAPE;
  if (n_plain > 0 && Y != nullptr && (ldy < n_plain || ldy % 8 != 0)) return W4A4_ERR_SHAPE;
  if (swiglu && n_plain > 0 && Y == nullptr) return W4A4_ERR_NULL;  // the plain (unquantised) outputs
  int st = check_gemm_args(Xq, Xsf, t_x, U, M, N, K, Wq, Wsf, t_w, L2t, r, bias, epilogue, next_q, N);
  if (st != W4A4_OK || M == 0) return st;
  if (!next_sf || !next_t) return W4A4_ERR_NULL;
  if (!aligned16(next_sf) || reinterpret_cast<uintptr_t>(next_t) % 4 != 0 || (Y && !aligned16(Y)) ||
      (H && !aligned16(H)) || (next_inv_s && !aligned16(next_inv_s)) ||
      reinterpret_cast<uintptr_t>(next_amax) % 4 != 0)
    return W4A4_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  st = device_setup(&dev);
  if (st != W4A4_OK) return st;
  QuantNext qn;
  qn.q = next_q;
  qn.sf = next_sf;
  qn.t = next_t;
  qn.ldq = next_ldq;
  qn.K = next_K;
  qn.col = next_col;
  return launch_gemm_pair<PairQNext>(Xq, Xsf, t_x, U, M, N, K, Wq, Wsf, t_w, L2t, r, bias, epilogue, Y, ldy,
                                     next_inv_s, reinterpret_cast<unsigned*>(next_amax),
                                     static_cast<cudaStream_t>(stream), dev, n_plain, H, ldh, qn);
}

size_t fp8_quant_workspace_bytes(int64_t rows, int64_t cols) {
  if (rows < 0 || cols <= 0 || cols % 8 != 0 || cols > kFp8MaxCols) return 0;
  return sizeof(float) * kAmaxMaxBlocks;  // the tensor-amax partial maxima
}

int fp8_quantize(const void* X, int64_t rows, int64_t cols, int64_t ldx, int transpose, uint8_t* out, int64_t ldo,
                 float* scale, void* workspace, size_t workspace_bytes, void* stream) {
  if (transpose != 0 && transpose != 1) return W4A4_ERR_ARG;
  if (rows < 0 || cols <= 0 || cols % 8 != 0 || ldx < cols || ldx % 8 != 0 || rows > (int64_t(1) << 30) ||
      cols > kFp8MaxCols)
    return W4A4_ERR_SHAPE;
  if (transpose ? (rows % 16 != 0 || ldo < rows || ldo % 16 != 0) : (ldo < cols || ldo % 8 != 0))
    return W4A4_ERR_SHAPE;
  if (rows == 0) return W4A4_OK;  // empty tensor: nothing enqueued
  if (!X || !out || !scale) return W4A4_ERR_NULL;
  if (!aligned16(X) || !aligned16(out) || reinterpret_cast<uintptr_t>(scale) % 4 != 0 ||
      (workspace && !aligned16(workspace)))
    return W4A4_ERR_ALIGN;
  if (!workspace || workspace_bytes < fp8_quant_workspace_bytes(rows, cols)) return W4A4_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  int st = device_setup(&dev);
  if (st != W4A4_OK) return st;
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  float* partials = static_cast<float*>(workspace);
  // pass 1: the tensor amax (column-segment CTAs times row bands, as for the activations)
  const int64_t gx = ceil_div(cols / 8, kAmaxThreads);
  int64_t gy = ceil_div(4 * static_cast<int64_t>(dev->num_sms), gx);
  if (gy > kAmaxMaxBlocks / gx) gy = kAmaxMaxBlocks / gx;
  if (gy > rows) gy = rows;
  if (gy < 1) gy = 1;
  const int64_t rows_per = ceil_div(rows, gy);
  gy = ceil_div(rows, rows_per);
  amax_kernel<__nv_bfloat16><<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)), kAmaxThreads, 0, strm>>>(
      static_cast<const __nv_bfloat16*>(X), rows, cols, ldx, nullptr, partials, static_cast<int>(rows_per));
  if (cudaGetLastError() != cudaSuccess) return W4A4_ERR_CUDA;
  // pass 2: codes, 128 x 64 tiles
  Fp8QuantParams p;
  p.X = static_cast<const __nv_bfloat16*>(X);
  p.rows = rows;
  p.cols = cols;
  p.ldx = ldx;
  p.out = out;
  p.ldo = ldo;
  p.partials = partials;
  p.n_partials = static_cast<int>(gx * gy);
  p.scale_out = scale;
  p.transpose = transpose;
  const int64_t ty = ceil_div(rows, 128);
  if (ty > 65535) return W4A4_ERR_SHAPE;
  fp8_quant_kernel<<<dim3(static_cast<unsigned>(ceil_div(cols, 64)), static_cast<unsigned>(ty)), 256, 0, strm>>>(p);
  if (cudaGetLastError() != cudaSuccess) return W4A4_ERR_CUDA;
  return W4A4_OK;
}

int attention_fp8(const uint8_t* Q8, const uint8_t* K8, const uint8_t* Vt8, int64_t batch, int64_t S, int64_t heads,
                  int64_t ldq, int64_t ldk, int64_t ldvt, const float* s_q, const float* s_k, const float* s_v,
                  float softmax_scale, void* O, int64_t ldo, void* stream) {
  if (batch < 0 || S < 0 || heads <= 0 || S % kAttnTile != 0 || heads > 65535 || batch > 65535 ||
      S > (int64_t(1) << 24) || batch * S > (int64_t(1) << 30) || heads * kAttnD > (int64_t(1) << 30))
    return W4A4_ERR_SHAPE;  // (token and feature coordinates stay 32-bit)
  const int64_t width = heads * kAttnD;
  if (ldq < width || ldq % 16 != 0 || ldk < width || ldk % 16 != 0 || ldvt < batch * S || ldvt % 16 != 0 ||
      ldo < width || ldo % 8 != 0)
    return W4A4_ERR_SHAPE;
  if (!(softmax_scale > 0.0f) || !(softmax_scale < 3.0e38f)) return W4A4_ERR_ARG;
  if (batch == 0 || S == 0) return W4A4_OK;  // no tokens
  if (!Q8 || !K8 || !Vt8 || !s_q || !s_k || !s_v || !O) return W4A4_ERR_NULL;
  if (!aligned16(Q8) || !aligned16(K8) || !aligned16(Vt8) || !aligned16(O) ||
      reinterpret_cast<uintptr_t>(s_q) % 4 != 0 || reinterpret_cast<uintptr_t>(s_k) % 4 != 0 ||
      reinterpret_cast<uintptr_t>(s_v) % 4 != 0)
    return W4A4_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  int st = device_setup(&dev);
  if (st != W4A4_OK) return st;
  CUtensorMap tq, tk, tv;
  if (!encode_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, Q8, static_cast<uint64_t>(width),
                 static_cast<uint64_t>(batch * S), static_cast<uint64_t>(ldq), 128u, 128u,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, K8, static_cast<uint64_t>(width),
                 static_cast<uint64_t>(batch * S), static_cast<uint64_t>(ldk), 128u, 128u,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, Vt8, static_cast<uint64_t>(batch * S),
                 static_cast<uint64_t>(width), static_cast<uint64_t>(ldvt), 128u, 128u,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return W4A4_ERR_CUDA;
  AttnParams p;
  p.S = static_cast<int>(S);
  p.heads = static_cast<int>(heads);
  p.s_q = s_q;
  p.s_k = s_k;
  p.s_v = s_v;
  p.scale = softmax_scale;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.ldo = ldo;
  p.status = dev->status_ptr;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(S / kAttnTile), static_cast<unsigned>(heads), static_cast<unsigned>(batch));
  cfg.blockDim = dim3(kAttnThreads, 1, 1);
  cfg.dynamicSmemBytes = AttnSmem::kBytes;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // set-up overlaps the previous kernel
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, attn_fp8_kernel, tq, tk, tv, p) != cudaSuccess) {
    cudaGetLastError();
    return W4A4_ERR_CUDA;
  }
  return W4A4_OK;
}

int w4a4_fp4_mma_rate(int iters, int pair, unsigned long long* cycles, void* stream) {
  if (iters < 1 || iters > (1 << 20)) return W4A4_ERR_SHAPE;
  if (pair != 0 && pair != 1) return W4A4_ERR_ARG;
  if (!cycles) return W4A4_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(cycles) % 8 != 0) return W4A4_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  int st = device_setup(&dev);
  if (st != W4A4_OK) return st;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(pair ? 2 * (dev->num_sms / 2) : dev->num_sms), 1, 1);
  cfg.blockDim = dim3(kRateThreads, 1, 1);
  cfg.dynamicSmemBytes = kRateSmem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = pair ? 2 : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pair ? 1 : 0;
  const cudaError_t e = pair ? cudaLaunchKernelEx(&cfg, fp4_mma_rate_kernel<true>, iters, cycles, dev->status_ptr)
                             : cudaLaunchKernelEx(&cfg, fp4_mma_rate_kernel<false>, iters, cycles, dev->status_ptr);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return W4A4_ERR_CUDA;
  }
  return W4A4_OK;
}

int w4a4_linear(const void* X, int64_t M, int64_t N, int64_t K, const uint8_t* Wq, const uint8_t* Wsf,
                const float* t_w, const float* inv_s, const void* L1t, const void* L2t, int r, const void* bias,
                int epilogue, void* Y, void* workspace, size_t workspace_bytes, void* stream) {
  if (M < 0 || N <= 0 || N % 8 != 0 || !valid_k(K) || M > (int64_t(1) << 30)) return W4A4_ERR_SHAPE;
  if (r != 0 && r != 16 && r != 32) return W4A4_ERR_SHAPE;
  if (!valid_lowrank_rows(M, r)) return W4A4_ERR_SHAPE;
  if (epilogue != W4A4_EPI_NONE && epilogue != W4A4_EPI_GELU_TANH) return W4A4_ERR_ARG;
  if (M == 0) return W4A4_OK;  // empty problem
  if (!X || !Wq || !Wsf || !t_w || !Y) return W4A4_ERR_NULL;
  if (r > 0 && (!L1t || !L2t)) return W4A4_ERR_NULL;
  if (!workspace || workspace_bytes < w4a4_workspace_bytes(M, N, K, r)) return W4A4_ERR_WORKSPACE;
  if (!aligned16(workspace)) return W4A4_ERR_ALIGN;
  const QuantPlan plan = quant_plan(M, K, r);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  size_t off = plan.bytes;
  uint8_t* Xq = w + off;
  off += round256(static_cast<size_t>(M) * static_cast<size_t>(K / 2));
  uint8_t* Xsf = w + off;
  off += round256(nvfp4_sf_bytes(M, K));
  float* t_x = reinterpret_cast<float*>(w + off);
  off += 256;
  void* U = r > 0 ? static_cast<void*>(w + off) : nullptr;
  int st = nvfp4_quantize_act(X, M, K, K, inv_s, L1t, r, t_w, Xq, Xsf, t_x, U, workspace, plan.bytes, stream);
  if (st != W4A4_OK) return st;
  return w4a4_gemm(Xq, Xsf, t_x, U, M, N, K, Wq, Wsf, t_w, L2t, r, bias, epilogue, Y, N, stream);
}

int nvfp4_sf_to_rowmajor(const uint8_t* sf_atoms, int64_t rows, int64_t K, uint8_t* sf_rowmajor, void* stream) {
  if (rows < 0 || !valid_k(K) || rows > (int64_t(1) << 30)) return W4A4_ERR_SHAPE;
  if (rows == 0) return W4A4_OK;
  if (!sf_atoms || !sf_rowmajor) return W4A4_ERR_NULL;
  if (!aligned16(sf_atoms) || !aligned16(sf_rowmajor)) return W4A4_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  const int st = device_setup(&dev);
  if (st != W4A4_OK) return st;
  const int64_t n = rows * (K / kQChunk);
  const int64_t blocks = ceil_div(n, 256);
  if (blocks > INT32_MAX) return W4A4_ERR_SHAPE;  // one grid dimension
  sf_to_rowmajor_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      sf_atoms, rows, K / kQChunk, sf_rowmajor);
  if (cudaGetLastError() != cudaSuccess) return W4A4_ERR_CUDA;
  return W4A4_OK;
}


}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free activation quantisation.  Its scratch is this file-scope
// device array; host code cannot use the symbol as a device address, so the
// address is looked up with cudaGetSymbolAddress, with the device current.
static __device__ __align__(256) uint8_t g_noalloc_scratch[W4A4_NOALLOC_SCRATCH_BYTES];

namespace {
// Per device: the address of the array whose zeroing has been enqueued
// (nullptr: not yet, or cleared again by w4a4_device_status with reset).
void* g_noalloc_zeroed[w4a4::kMaxDevices] = {};
std::mutex g_noalloc_mu;

int current_device_index() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= w4a4::kMaxDevices) {
    cudaGetLastError();
    return -1;
  }
  return dev;
}

// Device address of g_noalloc_scratch on the current device, or nullptr on
// failure.  The address is looked up on every call (a new context on the
// device loads the module again, possibly elsewhere); the first call for an
// address zeroes the array on ``stream`` (its counters must start at zero,
// and the kernels leave them zero).
void* noalloc_scratch(cudaStream_t stream) {
  const int dev = current_device_index();
  if (dev < 0) return nullptr;
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_zeroed[dev] != ptr) {
    if (cudaMemsetAsync(ptr, 0, W4A4_NOALLOC_SCRATCH_BYTES, stream) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_noalloc_zeroed[dev] = ptr;
  }
  return ptr;
}

// After a device error: the next no-alloc call on the current device zeroes
// the array again before it runs.
void noalloc_mark_dirty() {
  const int dev = current_device_index();
  if (dev < 0) return;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  g_noalloc_zeroed[dev] = nullptr;
}
}  // namespace

extern "C" {

int nvfp4_quantize_act_noalloc(const void* X, int64_t M, int64_t K, int64_t ldx, const float* inv_s, const void* L1t,
                               int r, const float* t_w, uint8_t* Xq, uint8_t* Xsf, float* t_x, void* U,
                               void* stream) {
  if (M < 0 || !valid_k(K) || ldx < K || ldx % 8 != 0 || M > (int64_t(1) << 30)) return W4A4_ERR_SHAPE;
  if (r != 0 && r != 16 && r != 32) return W4A4_ERR_SHAPE;
  if (!valid_lowrank_rows(M, r)) return W4A4_ERR_SHAPE;
  if (M == 0) return W4A4_OK;  // empty problem
  const size_t need = nvfp4_quant_workspace_bytes(M, K, r);
  if (need > W4A4_NOALLOC_SCRATCH_BYTES) return W4A4_ERR_SCRATCH_LIMIT;
  if (!X || !Xq || !Xsf || !t_x) return W4A4_ERR_NULL;
  if (r > 0 && (!L1t || !t_w || !U)) return W4A4_ERR_NULL;
  DeviceInfo* dev = nullptr;
  int st = device_setup(&dev);
  if (st != W4A4_OK) return st;
  void* scratch = noalloc_scratch(static_cast<cudaStream_t>(stream));
  if (scratch == nullptr) return W4A4_ERR_CUDA;
  return nvfp4_quantize_act(X, M, K, ldx, inv_s, L1t, r, t_w, Xq, Xsf, t_x, U, scratch,
                            W4A4_NOALLOC_SCRATCH_BYTES, stream);
}

int w4a4_device_status(int* status, int reset) {
  if (!status) return W4A4_ERR_NULL;
  if (cudaDeviceSynchronize() != cudaSuccess) { cudaGetLastError(); return W4A4_ERR_CUDA; }
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) { cudaGetLastError(); return W4A4_ERR_CUDA; }
  *status = v;
  if (reset) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) { cudaGetLastError(); return W4A4_ERR_CUDA; }
    noalloc_mark_dirty();
  }
  return W4A4_OK;
}

int w4a4_last_error(void) {
  // the sticky status word as it stands, read on a private non-blocking
  // stream: no wait for the caller's work (the caller synchronises first)
  static cudaStream_t reader[kMaxDevices] = {};
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) {
    cudaGetLastError();
    return W4A4_ERR_CUDA;
  }
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!reader[d] && cudaStreamCreateWithFlags(&reader[d], cudaStreamNonBlocking) != cudaSuccess) {
      cudaGetLastError();
      reader[d] = nullptr;
      return W4A4_ERR_CUDA;
    }
  }
  int v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_status, sizeof(int), 0, cudaMemcpyDeviceToHost, reader[d]) != cudaSuccess ||
      cudaStreamSynchronize(reader[d]) != cudaSuccess) {
    cudaGetLastError();
    return W4A4_ERR_CUDA;
  }
  return v;
}

int w4a4_set_wait_bound(int64_t cycles) {
  if (cycles <= 0) cycles = kDefaultWaitBoundCycles;
  if (cycles < 1000000) return W4A4_ERR_ARG;
  DeviceInfo* dev = nullptr;
  const int st = device_setup(&dev);
  if (st != W4A4_OK) return st;
  const long long v = cycles;
  if (cudaDeviceSynchronize() != cudaSuccess || cudaMemcpyToSymbol(c_wait_bound_cycles, &v, sizeof(v)) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return W4A4_ERR_CUDA;
  }
  return W4A4_OK;
}

const char* w4a4_status_string(int status) {
  switch (status) {
    case W4A4_OK: return "ok";
    case W4A4_ERR_NULL: return "a required pointer is NULL";
    case W4A4_ERR_SHAPE: return "unsupported size or rank";
    case W4A4_ERR_ALIGN: return "pointer or leading dimension not 16-byte aligned";
    case W4A4_ERR_ARCH: return "no CUDA device of compute capability 10.x (sm_100a) is current";
    case W4A4_ERR_WORKSPACE: return "workspace missing or too small";
    case W4A4_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case W4A4_ERR_DEVICE_TIMEOUT: return "a device-side pipeline wait exceeded its bound";
    case W4A4_ERR_ARG: return "an enum argument is out of range";
    case W4A4_ERR_SCRATCH_LIMIT: return "the problem needs more scratch than the built-in no-alloc array holds";
    case W4A4_ERR_DEVICE_LAYOUT: return "a kernel found its dynamic shared memory base misaligned";
    default: return "unknown status";
  }
}

}  // extern "C"
