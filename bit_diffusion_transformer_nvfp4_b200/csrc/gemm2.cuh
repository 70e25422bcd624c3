// gemm2.cuh -- the W4A4 GEMM on CTA pairs (tcgen05 cta_group::2).
//
// Same computation as gemm.cuh (block-scaled FP4 main product, hi|lo
// low-rank pass into the same fp32 TMEM accumulator, bias / GELU / bf16
// epilogue), restructured so that two SMs share one 256 x BN output tile:
//
//   * each CTA of the pair TMA-loads its own 128 rows of A (activation codes),
//     its own half (BN/2 rows) of B (weight codes), its 128 rows' scale atoms
//     and all BN rows' weight scale atoms; the loads of both CTAs complete on
//     the even CTA's ring barrier;
//   * the even CTA's MMA thread issues M=256 MMAs that read A and B from both
//     CTAs' shared memory, so per SM the shared-memory traffic per FLOP is
//     about half that of a single-CTA 128 x 256 tile;
//   * block scales bypass the tensor pipe: tcgen05.cp copies execute in the
//     same in-order queue as the MMAs (twelve per 256-deep K step cost about
//     as much as the four MMAs), so instead each CTA's scale atoms travel
//     through their own small shared-memory ring, loaded several K steps
//     ahead, and four scale warps per CTA (one per TMEM lane quarter) write
//     them into a ring of TMEM scale slots with tcgen05.st; the MMA thread
//     waits for a slot's eight warp arrivals and frees it with a multicast
//     commit;
//   * ring stages and the accumulator are handed back with multicast
//     tcgen05.commit to both CTAs; the odd CTA's epilogue releases the
//     accumulator with remote mbarrier arrives;
//   * the epilogue stages bf16 results in 64-byte-swizzled shared memory and
//     writes them with TMA stores (full 64-byte rows, clipped at the edges).
//
// One persistent CTA pair per two SMs; 512 threads per CTA: warp 0 A/B TMA
// producer, warp 1 TMEM owner (+ MMA issuer in the even CTA), warp 2 scale
// TMA producer, warp 3 spare, warps 4-7 scale warps, warps 8-15 epilogue.  The launch gives every
// thread 128 registers; setmaxnreg then shrinks the first two warpgroups and
// grows the two epilogue warpgroups, whose 128 accumulator columns per thread
// would otherwise spill.
#pragma once

#include "gemm.cuh"
#include "sm100.cuh"

namespace w4a4 {

template <int BN_, int STAGES_, int SF_STAGES_ = 5, int EPI_NBUF_ = 2, bool ALIGN_BASE_ = true, bool QNEXT_ = false,
          bool ROPE_ = false>
struct Gemm2Cfg {
  // QNEXT: the epilogue can also quantise its outputs for the next layer;
  // ROPE: it can rotate the leading plain outputs by the rotary embedding
  // (separate instantiations, so the plain GEMM keeps its registers)
  static constexpr bool QNEXT = QNEXT_;
  static constexpr bool ROPE = ROPE_;
  static constexpr int BN = BN_;                       // tile width (output columns)
  static constexpr int BH = BN / 2;                    // B rows held by each CTA
  static constexpr int STAGES = STAGES_;
  static constexpr int BM = 128;                       // rows per CTA (256 per pair)
  static constexpr int BK = 256;
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = BH * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int LR_BYTES = BM * 128 + BH * 64;  // U tile + this CTA's L2t half at rank 32 (rank 16: half)
  // scale ring: one slot per 256-deep K step, this CTA's 128 rows of A
  // scales (4 atoms) and the weight scales of every 128-row block the tile
  // touches (a 192-wide tile may start 64 rows into a block)
  static constexpr int SFA_BYTES = 4 * 512;
  static constexpr int SFB_RB = BN / 128 + (BN % 128 ? 1 : 0);
  static constexpr int SFB_BYTES = SFB_RB * 4 * 512;
  static constexpr int SF_STAGE_BYTES = SFA_BYTES + SFB_BYTES;
  static constexpr int SF_STAGES = SF_STAGES_;
  // TMEM: accumulator(s), then scale slots of SF_COLS columns (per K-block j
  // of the step: A scales at 4j, weight-scale block rb at 16 + 4*SFB_RB*j + 4*rb)
  static constexpr int SF_COLS = 16 + 4 * 4 * SFB_RB;
  static constexpr int NUM_ACC = (2 * BN + 2 * SF_COLS <= 512) ? 2 : 1;
  static constexpr int SF_COL0 = NUM_ACC * BN;
  static constexpr int NB_TSF_FIT = (512 - SF_COL0) / SF_COLS;
  static constexpr int NB_TSF = NB_TSF_FIT < 6 ? NB_TSF_FIT : 6;
  static constexpr int TMEM_COLS = 512;
  static constexpr int EPI_WARPS = 8;
  static constexpr int SF_WARP0 = 4;                   // warps 4-7: scale warps
  static constexpr int EPI_WARP0 = 8;                  // warps 8-15: epilogue
  static constexpr int THREADS = 32 * (EPI_WARP0 + EPI_WARPS);
  // registers per thread after setmaxnreg: producer / MMA warpgroup, scale
  // warpgroup, the two epilogue warpgroups (launch: 65536 / THREADS = 128);
  // the rotary epilogue holds the table values beside the accumulator's, so
  // its instantiation moves 8 registers from each of the first two to them
  static constexpr int REGS_CTRL = ROPE ? 56 : 64, REGS_SF = ROPE ? 56 : 64, REGS_EPI = ROPE ? 184 : 176;
  static constexpr int HALF = BN / 2;                  // columns per epilogue warp
  static constexpr int EPI_BUF = 32 * 64;              // 32 rows x 32 bf16, one staging buffer
  static constexpr int EPI_NBUF = EPI_NBUF_;           // staging buffers per epilogue warp
  static constexpr int EPI_BYTES = EPI_WARPS * EPI_NBUF * EPI_BUF;
  // ALIGN_BASE: round the dynamic shared memory base up to 1024 bytes (costs
  // up to 1 KB); otherwise the base must already be 1024-aligned (checked)
  static constexpr bool ALIGN_BASE = ALIGN_BASE_;
  // mbarriers (full/empty, accumulator, scale ring, TMEM scale slots, drain),
  // then the TMEM address and the abort flag
  static constexpr int BAR_BYTES = (8 * (2 * STAGES + 2 * 2 + 2 * SF_STAGES + 2 * 6 + 1) + 8 + 127) / 128 * 128;
  static constexpr int SMEM =
      STAGE_BYTES * STAGES + SF_STAGE_BYTES * SF_STAGES + EPI_BYTES + (ALIGN_BASE ? 1024 : 0) + BAR_BYTES;

  static_assert(NB_TSF >= 2 && SF_COL0 + NB_TSF * SF_COLS <= TMEM_COLS, "TMEM budget");
  static_assert(SF_COLS % 16 == 0, "scale slot written 16 columns at a time");
  static_assert(STAGE_BYTES % 1024 == 0 && SF_STAGE_BYTES % 1024 == 0, "stage alignment");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(BN % 64 == 0 && HALF % 32 == 0, "tile shape");
  static_assert(THREADS == 512, "four warpgroups");
  static_assert(128 * (REGS_CTRL + REGS_SF + 2 * REGS_EPI) <= 65536 - 4096,
                "register budgets fit the launch allocation with room to spare");
};

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    gemm2_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                 const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
                 const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_l2,
                 const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_h,
                 const GemmParams p) {
  constexpr int BN = C::BN, STAGES = C::STAGES;
  // the next kernel in the stream (a programmatic dependent) may be scheduled
  // on SMs this grid leaves; it waits for this grid's completion itself
  grid_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = C::ALIGN_BASE
                      ? reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023))
                      : smem_raw;
  if (!C::ALIGN_BASE && (smem_u32(smem_raw) & 1023u) != 0) {
    // the swizzled TMA tiles need 1024-byte alignment; every CTA sees the
    // same base, so all return here before any barrier or TMEM use
    if (threadIdx.x == 0 && p.status) atomicExch(p.status, kStatusMisaligned);
    return;
  }
  uint8_t* sf_smem = smem + C::STAGE_BYTES * STAGES;
  uint8_t* epi_smem = sf_smem + C::SF_STAGE_BYTES * C::SF_STAGES;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_smem + C::EPI_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + C::NUM_ACC;
  uint64_t* sf_full = acc_empty + C::NUM_ACC;     // [SF_STAGES] this CTA's scale atoms landed
  uint64_t* sf_empty = sf_full + C::SF_STAGES;    // [SF_STAGES] the scale warps have read them
  uint64_t* tsf_ready = sf_empty + C::SF_STAGES;  // [NB_TSF] even CTA's: both CTAs' slot written
  uint64_t* tsf_free = tsf_ready + C::NB_TSF;     // [NB_TSF] the MMAs that read the slot are done
  uint64_t* drain = tsf_free + C::NB_TSF;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const bool lr = p.has_lr != 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < C::NUM_ACC; ++a) {
      mbar_init(smem_u32(&acc_full[a]), 1);
      mbar_init(smem_u32(&acc_empty[a]), 2 * C::EPI_WARPS);
    }
    for (int s = 0; s < C::SF_STAGES; ++s) {
      mbar_init(smem_u32(&sf_full[s]), 1);
      mbar_init(smem_u32(&sf_empty[s]), 4);
    }
    for (int b = 0; b < C::NB_TSF; ++b) {
      mbar_init(smem_u32(&tsf_ready[b]), 8);
      mbar_init(smem_u32(&tsf_free[b]), 1);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_sfa);
    tma_prefetch_desc(&tm_sfb);
    tma_prefetch_desc(&tm_y);
    if (p.n_plain < p.N) tma_prefetch_desc(&tm_h);
    if (lr) {
      tma_prefetch_desc(&tm_u);
      tma_prefetch_desc(&tm_l2);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers are initialised before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // set-up above overlaps the tail of the previous kernel in the stream
  // (programmatic launch); nothing below may touch memory before this
  grid_dependency_wait();

  const int m_tiles = (p.M + 2 * C::BM - 1) / (2 * C::BM);
  const int n_tiles = (p.N + BN - 1) / BN;
  const int total = m_tiles * n_tiles;
  const int nkb = (p.K + C::BK - 1) / C::BK;  // the last K step may be partial: TMA fills zeros
  const int pair = blockIdx.x >> 1;
  const int pairs = gridDim.x >> 1;
  // K steps (with scales) this pair runs: every tile pair, pair+pairs, ...
  const uint32_t total_ks = pair < total ? static_cast<uint32_t>((total - 1 - pair) / pairs + 1) * nkb : 0u;

  // Registers: each role sets its warpgroup's budget first thing (the
  // control and scale warpgroups give theirs back, the epilogue warpgroups
  // take them), inside its own branch so that the compiler allocates each
  // role's code to its budget.
  if (warp < C::SF_WARP0) regs_release_to<C::REGS_CTRL>();
  // scale atoms of K step k (counted over this pair's tiles) into slot k % SF_STAGES
  auto issue_sf = [&](uint32_t k) -> bool {
    const int tile = pair + static_cast<int>(k / nkb) * pairs;
    const int kb = static_cast<int>(k % nkb);
    const int m0 = (tile % m_tiles) * 2 * C::BM + static_cast<int>(rank) * C::BM;
    const int n0 = (tile / m_tiles) * BN;
    const uint32_t slot = k % C::SF_STAGES;
    if (k >= static_cast<uint32_t>(C::SF_STAGES) &&
        !mbar_wait(smem_u32(&sf_empty[slot]), ((k / C::SF_STAGES) - 1) & 1, abort_flag, p.status))
      return false;
    uint8_t* dst = sf_smem + slot * C::SF_STAGE_BYTES;
    const uint32_t bar = smem_u32(&sf_full[slot]);
    mbar_arrive_expect_tx(bar, C::SF_STAGE_BYTES);
    tma_load_3d(smem_u32(dst), &tm_sfa, bar, 0, kb * 4, m0 / 128);
    tma_load_3d(smem_u32(dst + C::SFA_BYTES), &tm_sfb, bar, 0, kb * 4, n0 / 128);
    return true;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ A/B producer (both CTAs)
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += pairs) {
        const int m0 = (tile % m_tiles) * 2 * C::BM + static_cast<int>(rank) * C::BM;
        const int n0 = (tile / m_tiles) * BN;
        const int nb0 = n0 + static_cast<int>(rank) * C::BH;
        if (lr) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, abort_flag, p.status)) { ok = false; break; }
          uint8_t* st = smem + s * C::STAGE_BYTES;
          const uint32_t bar = mapa_shared(smem_u32(&full[s]), 0);
          if (leader) mbar_arrive_expect_tx(smem_u32(&full[s]), 2 * C::LR_BYTES * p.r / 32);
          tma_load_2d_pair(smem_u32(st), &tm_u, bar, 0, m0);
          tma_load_2d_pair(smem_u32(st + C::A_BYTES), &tm_l2, bar, 0, nb0);
          ++it;
        }
        for (int kb = 0; kb < nkb; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, abort_flag, p.status)) { ok = false; break; }
          uint8_t* st = smem + s * C::STAGE_BYTES;
          const uint32_t bar = mapa_shared(smem_u32(&full[s]), 0);
          if (leader) mbar_arrive_expect_tx(smem_u32(&full[s]), 2 * C::STAGE_BYTES);
          tma_load_2d_pair(smem_u32(st), &tm_a, bar, kb * 128, m0);
          tma_load_2d_pair(smem_u32(st + C::A_BYTES), &tm_b, bar, kb * 128, nb0);
          ++it;
        }
      }
      // The even CTA's ring barriers count both CTAs' bytes: there, wait
      // (bounded) for the newest fills to land before shared memory goes away.
      if (leader) {
        const uint32_t first = it > static_cast<uint32_t>(STAGES) ? it - STAGES : 0u;
        for (uint32_t j = first; j < it; ++j) mbar_wait_drain(smem_u32(&full[j % STAGES]), (j / STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (leader && lane == 0) {
      constexpr uint32_t kIdescF4 = idesc_nvf4(256, BN);
      constexpr uint32_t kIdescBf = idesc_bf16(256, BN);
      uint32_t it = 0, tcount = 0, ks = 0;
      for (int tile = pair; tile < total; tile += pairs) {
        const uint32_t acc = tcount % C::NUM_ACC;
        const uint32_t aph = (tcount / C::NUM_ACC) & 1;
        if (!mbar_wait(smem_u32(&acc_empty[acc]), aph ^ 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        // a tile starting 64 rows into a weight-scale block reads its scales
        // two TMEM columns further on
        const uint32_t sfb_shift = static_cast<uint32_t>(((tile / m_tiles) * BN % 128) / 32);
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
            if (k < p.r / 8)
              mma_bf16_pair(d, lowrank_desc_u(a_base, k, p.r), lowrank_desc_l2(b_base, k, p.r), kIdescBf, k > 0 ? 1u : 0u);
          }
          tc_commit_pair_mc(smem_u32(&empty[s]), 0x3);
          ++it;
          first = false;
        }
        for (int kb = 0; kb < nkb; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(smem_u32(&full[s]), ph, abort_flag, p.status)) { ok = false; break; }
          const uint32_t b = ks % C::NB_TSF;
          if (!mbar_wait(smem_u32(&tsf_ready[b]), (ks / C::NB_TSF) & 1, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + s * C::STAGE_BYTES);
          const uint32_t b_base = a_base + C::A_BYTES;
          const uint32_t sf = tmem + C::SF_COL0 + b * C::SF_COLS;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t ad = smem_desc(a_base + 32 * j, 16, 1024, kSwizzle128B);
            const uint64_t bd = smem_desc(b_base + 32 * j, 16, 1024, kSwizzle128B);
            mma_nvf4_pair(d, ad, bd, kIdescF4, sf + 4 * j, sf + 16 + 4 * C::SFB_RB * j + sfb_shift,
                          (!first || j > 0) ? 1u : 0u);
          }
          tc_commit_pair_mc(smem_u32(&empty[s]), 0x3);
          tc_commit_pair_mc(smem_u32(&tsf_free[b]), 0x3);
          ++it;
          ++ks;
          first = false;
        }
        if (!ok) break;
        tc_commit_pair_mc(smem_u32(&acc_full[acc]), 0x3);
        ++tcount;
      }
      tc_commit_pair(smem_u32(drain));
      mbar_wait_drain(smem_u32(drain), 0);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ scale-ring producer (both CTAs)
    // Its own thread, so that a slot the scale warps have not yet freed never
    // holds up the A/B stages.
    if (lane == 0) {
      uint32_t ksf = 0;
      while (ksf < total_ks && issue_sf(ksf)) ++ksf;
      // no scale copy may still be landing when shared memory goes away
      const uint32_t sf_first = ksf > static_cast<uint32_t>(C::SF_STAGES) ? ksf - C::SF_STAGES : 0u;
      for (uint32_t k = sf_first; k < ksf; ++k)
        mbar_wait_drain(smem_u32(&sf_full[k % C::SF_STAGES]), (k / C::SF_STAGES) & 1);
    }
  } else if (warp < C::SF_WARP0) {
    // spare warp
  } else if (warp >= C::EPI_WARP0) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    regs_grow_to<C::REGS_EPI>();
    const int ew = warp - C::EPI_WARP0;
    const int q = warp & 3;               // TMEM lane quarter (rows 32q..32q+31 of this CTA)
    const int h = ew >> 2;                // column half
    const float alpha = __fmul_rn(__ldg(p.t_x), __ldg(p.t_w));
    // the next layer's tensor scale, when this epilogue quantises for it
    const float t_next = C::QNEXT && p.q_next != nullptr ? __ldg(p.t_next) : 1.0f;
    const float rt_next = __frcp_rn(t_next);
    const uint32_t acc_empty_leader0 = mapa_shared(smem_u32(&acc_empty[0]), 0);
    uint8_t* stage_buf = epi_smem + ew * C::EPI_NBUF * C::EPI_BUF;
    float amax = 0.0f;  // next layer's amax over this thread's stored outputs
    uint32_t tcount = 0, chunk = 0;
    for (int tile = pair; tile < total; tile += pairs) {
      const int m0 = (tile % m_tiles) * 2 * C::BM + static_cast<int>(rank) * C::BM;
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
      if (lane == 0) mbar_arrive_cluster(acc_empty_leader0 + 8 * acc);

      const int row0 = m0 + q * 32;
      // the staging buffer of the next 32 x 32 output box, once the TMA store
      // that last used it has finished reading it
      auto next_buf = [&]() -> uint8_t* {
        uint8_t* buf = stage_buf + (chunk % C::EPI_NBUF) * C::EPI_BUF;
        if (chunk >= static_cast<uint32_t>(C::EPI_NBUF)) {
          if (lane == 0) bulk_wait_group_read<C::EPI_NBUF - 1>();
          __syncwarp();
        }
        return buf;
      };
      // row `lane` of a 32 x 32 bf16 box, 64-byte rows, 64-byte swizzle
      auto stage_row = [&](uint8_t* buf, const uint32_t (&packed)[16]) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int phys = g ^ ((lane >> 1) & 3);
          *reinterpret_cast<uint4*>(buf + lane * 64 + phys * 16) =
              make_uint4(packed[4 * g], packed[4 * g + 1], packed[4 * g + 2], packed[4 * g + 3]);
        }
      };
      // next layer's amax over a staged box (only outputs the TMA store
      // keeps: rows < M, columns < ncols).  Lane l takes columns 2(l%16),
      // 2(l%16)+1 of rows 16(l/16) .. +15: packed maxima of |y| down the
      // column pair, then one multiply by the next 1/s per column.
      auto fold_amax = [&](const uint8_t* buf, int col0, int ncols) {
        __syncwarp();
        const int cpair = lane & 15;
        const int rbase = (lane >> 4) * 16;
        uint32_t mx = 0u;
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
          const int row = rbase + rr;
          if (row0 + row < p.M) {
            const int phys = (cpair >> 2) ^ ((row >> 1) & 3);
            mx = bf16x2_absmax(mx, *reinterpret_cast<const uint32_t*>(buf + row * 64 + phys * 16 + (cpair & 3) * 4));
          }
        }
        const int col = col0 + 2 * cpair;
        if (col < ncols) {  // ncols % 8 == 0: both columns of the pair are valid
          float v0 = bf16_lo(mx & 0x7FFF7FFFu), v1 = bf16_hi(mx & 0x7FFF7FFFu);
          if (p.next_inv_s != nullptr) {
            const float2 s2 = __ldg(reinterpret_cast<const float2*>(p.next_inv_s + col));
            v0 = __fmul_rn(v0, s2.x);
            v1 = __fmul_rn(v1, s2.y);
          }
          amax = fmaxf(amax, fmaxf(v0, v1));
        }
      };
      // the next layer's NVFP4 codes and scale bytes of the 32 outputs of
      // this row in ``pk`` (output columns col .. col+31: two 16-blocks),
      // the same arithmetic as the activation quantiser under the given t
      auto quant_next = [&](const uint32_t (&pk)[16], int col, int ncols) {
        const int row = row0 + lane;
        if (row >= p.M || col >= ncols) return;  // ncols % 32 == 0: the 32 columns are all valid
        float x[32];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          x[2 * j] = bf16_lo(pk[j]);
          x[2 * j + 1] = bf16_hi(pk[j]);
        }
        if (p.next_inv_s != nullptr) {
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const float4 s4 = __ldg(reinterpret_cast<const float4*>(p.next_inv_s + col + j));
            x[j] = __fmul_rn(x[j], s4.x);
            x[j + 1] = __fmul_rn(x[j + 1], s4.y);
            x[j + 2] = __fmul_rn(x[j + 2], s4.z);
            x[j + 3] = __fmul_rn(x[j + 3], s4.w);
          }
        }
        // two blocks' scale bytes in one conversion; byte 0 = the first block
        const uint32_t e2 = cvt_e4m3x2(div6(__fmul_rn(absmax16(x + 16), rt_next)),
                                       div6(__fmul_rn(absmax16(x), rt_next))) & 0xFFFFu;
        uint32_t cw[4];
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
          const uint32_t e = (e2 >> (8 * q2)) & 0xFFu;
          const float rq = __frcp_rn(__fmul_rn(e4m3x2_to_f32(e).y, t_next));  // 1/(dec(e) t)
#pragma unroll
          for (int uu = 0; uu < 2; ++uu) {
            float v[8];
#pragma unroll
            for (int jj = 0; jj < 8; jj += 2)
              mul2_rn(v[jj], v[jj + 1], x[16 * q2 + 8 * uu + jj], x[16 * q2 + 8 * uu + jj + 1], rq, rq);
            cw[2 * q2 + uu] = e != 0u ? cvt_e2m1x8(v) : 0u;  // a zero scale leaves the codes +0
          }
        }
        const int kcol = p.q_col0 + col;  // column in the next layer's activation (multiple of 32)
        *reinterpret_cast<uint4*>(p.q_next + static_cast<int64_t>(row) * p.ldq + kcol / 2) =
            make_uint4(cw[0], cw[1], cw[2], cw[3]);
        const int64_t atom = static_cast<int64_t>(row / 128) * (p.next_K / 64) + kcol / 64;
        *reinterpret_cast<uint16_t*>(p.sf_next + atom * 512 + (row % 32) * 16 + ((row / 32) % 4) * 4 + (kcol / 16) % 4) =
            static_cast<uint16_t>(e2);
      };
      if (n0 < p.n_plain) {
        // ---------------------------------------------------- plain outputs
#pragma unroll
        for (int c = 0; c < C::HALF / 32; ++c, ++chunk) {
          const int n = n0 + h * C::HALF + 32 * c;
          // rotary embedding of this block (32 features of one head): the
          // (cos, sin) of its 16 pairs for this thread's token, 128 bytes of
          // the token's table row, read eight values per group of outputs
          // (a whole block's 32 would not fit beside the accumulator values
          // without spilling); rows past M read the last row (their outputs
          // are dropped by the store)
          const bool rot = C::ROPE && n < p.n_rope;  // the same for the whole warp
          const float4* src = nullptr;
          if constexpr (C::ROPE)
            src = reinterpret_cast<const float4*>(p.rope + static_cast<int64_t>(min(row0 + lane, p.M - 1)) * p.ld_rope +
                                                  n % p.d_head);
          uint8_t* buf = next_buf();
          uint32_t packed[16];
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            float cs[8];
            if constexpr (C::ROPE) {
              if (rot) {
                const float4 v0 = __ldg(src + 2 * g), v1 = __ldg(src + 2 * g + 1);
                cs[0] = v0.x; cs[1] = v0.y; cs[2] = v0.z; cs[3] = v0.w;
                cs[4] = v1.x; cs[5] = v1.y; cs[6] = v1.z; cs[7] = v1.w;
              }
            }
            float b[8];
            if (p.bias != nullptr && n + 8 * g < p.n_plain) {
              const uint4 bw = __ldg(reinterpret_cast<const uint4*>(p.bias + n + 8 * g));
              b[0] = bf16_lo(bw.x); b[1] = bf16_hi(bw.x); b[2] = bf16_lo(bw.y); b[3] = bf16_hi(bw.y);
              b[4] = bf16_lo(bw.z); b[5] = bf16_hi(bw.z); b[6] = bf16_lo(bw.w); b[7] = bf16_hi(bw.w);
            } else {
#pragma unroll
              for (int j = 0; j < 8; ++j) b[j] = 0.0f;
            }
#pragma unroll
            for (int j = 0; j < 8; j += 2) {
              float y0 = __fadd_rn(__fmul_rn(alpha, __uint_as_float(r[32 * c + 8 * g + j])), b[j]);
              float y1 = __fadd_rn(__fmul_rn(alpha, __uint_as_float(r[32 * c + 8 * g + j + 1])), b[j + 1]);
              if (!C::ROPE && p.epi == 1) {  // (the rotary entry point has no GELU)
                y0 = gelu_tanh_f32(y0);
                y1 = gelu_tanh_f32(y1);
              }
              if constexpr (C::ROPE) {
                if (rot) {
                  // pair (8g + j) / 2 of the block: (y0, y1) turned by its angle
                  const float co = cs[j], si = cs[j + 1];
                  const float r0 = __fmaf_rn(y0, co, -__fmul_rn(y1, si));
                  const float r1 = __fmaf_rn(y0, si, __fmul_rn(y1, co));
                  y0 = r0;
                  y1 = r1;
                }
              }
              packed[4 * g + j / 2] = pack_bf16x2(y0, y1);
            }
          }
          stage_row(buf, packed);
          if (p.next_amax != nullptr && p.n_plain == p.N) fold_amax(buf, n, p.N);
          if constexpr (C::QNEXT) {
            if (p.q_next != nullptr && p.n_plain == p.N) quant_next(packed, n, p.N);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && p.Y != nullptr) {
            tma_store_2d(&tm_y, smem_u32(buf), n, row0);
            bulk_commit_group();
          }
        }
      } else {
        // ---------------------------------------------------- SwiGLU pairs
        // Each 32-column accumulator block holds 16 gate and then the 16 up
        // features of the same outputs; two blocks fill one 32-column box of H.
        const int n_h = (p.N - p.n_plain) / 2;
        const int hc0 = (n0 - p.n_plain) / 2 + h * (C::HALF / 2);
#pragma unroll
        for (int c2 = 0; c2 < C::HALF / 64; ++c2, ++chunk) {
          uint8_t* buf = next_buf();
          uint32_t packed[16];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int c = 2 * c2 + hh;
            const int nw = n0 + h * C::HALF + 32 * c;  // first gate row of the block
            float bg[16], bu[16];
            if (p.bias != nullptr && nw < p.N) {  // (N - n_plain) % 32 == 0: the whole block is valid
#pragma unroll
              for (int v = 0; v < 2; ++v) {
                const uint4 gw = __ldg(reinterpret_cast<const uint4*>(p.bias + nw + 8 * v));
                const uint4 uw = __ldg(reinterpret_cast<const uint4*>(p.bias + nw + 16 + 8 * v));
                const uint32_t gg[4] = {gw.x, gw.y, gw.z, gw.w}, uu[4] = {uw.x, uw.y, uw.z, uw.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  bg[8 * v + 2 * j] = bf16_lo(gg[j]);
                  bg[8 * v + 2 * j + 1] = bf16_hi(gg[j]);
                  bu[8 * v + 2 * j] = bf16_lo(uu[j]);
                  bu[8 * v + 2 * j + 1] = bf16_hi(uu[j]);
                }
              }
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j) bg[j] = bu[j] = 0.0f;
            }
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              const float g0 = __fadd_rn(__fmul_rn(alpha, __uint_as_float(r[32 * c + j])), bg[j]);
              const float g1 = __fadd_rn(__fmul_rn(alpha, __uint_as_float(r[32 * c + j + 1])), bg[j + 1]);
              const float u0 = __fadd_rn(__fmul_rn(alpha, __uint_as_float(r[32 * c + 16 + j])), bu[j]);
              const float u1 = __fadd_rn(__fmul_rn(alpha, __uint_as_float(r[32 * c + 16 + j + 1])), bu[j + 1]);
              packed[8 * hh + j / 2] = pack_bf16x2(__fmul_rn(silu_f32(g0), u0), __fmul_rn(silu_f32(g1), u1));
            }
          }
          stage_row(buf, packed);
          const int hc = hc0 + 32 * c2;
          if (p.next_amax != nullptr) fold_amax(buf, hc, n_h);
          if constexpr (C::QNEXT) {
            if (p.q_next != nullptr) quant_next(packed, hc, n_h);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && p.H != nullptr) {
            tma_store_2d(&tm_h, smem_u32(buf), hc, row0);
            bulk_commit_group();
          }
        }
      }
      ++tcount;
    }
    if (p.next_amax != nullptr) amax_publish(amax, p.next_amax);
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  } else {
    // ------------------------------------------------------------ scale warps (both CTAs)
    regs_release_to<C::REGS_SF>();
    // Lane l holds, per 512-byte atom, the 16 bytes of rows l, l+32, l+64,
    // l+96 (one 32-bit TMEM column per row); every lane quarter gets the same
    // words, so each row's scales sit in its own lane at column 4j + row/32.
    const int q = warp & 3;  // the TMEM lane quarter this warp may write
    const uint32_t tsf_ready_leader0 = mapa_shared(smem_u32(&tsf_ready[0]), 0);
    for (uint32_t k = 0; k < total_ks; ++k) {
      const uint32_t slot = k % C::SF_STAGES;
      const uint32_t b = k % C::NB_TSF;
      if (!mbar_wait(smem_u32(&sf_full[slot]), (k / C::SF_STAGES) & 1, abort_flag, p.status)) break;
      if (k >= static_cast<uint32_t>(C::NB_TSF) &&
          !mbar_wait(smem_u32(&tsf_free[b]), ((k / C::NB_TSF) - 1) & 1, abort_flag, p.status))
        break;
      const uint8_t* src = sf_smem + slot * C::SF_STAGE_BYTES;
      uint32_t v[C::SF_COLS];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 w = *reinterpret_cast<const uint4*>(src + 512 * j + 16 * lane);
        v[4 * j] = w.x; v[4 * j + 1] = w.y; v[4 * j + 2] = w.z; v[4 * j + 3] = w.w;
#pragma unroll
        for (int rb = 0; rb < C::SFB_RB; ++rb) {
          const uint4 u = *reinterpret_cast<const uint4*>(src + C::SFA_BYTES + 2048 * rb + 512 * j + 16 * lane);
          const int c = 16 + 4 * C::SFB_RB * j + 4 * rb;
          v[c] = u.x; v[c + 1] = u.y; v[c + 2] = u.z; v[c + 3] = u.w;
        }
      }
      tc_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + C::SF_COL0 + b * C::SF_COLS;
#pragma unroll
      for (int c = 0; c < C::SF_COLS; c += 16)
        tmem_st_16cols(taddr + c, *reinterpret_cast<const uint32_t(*)[16]>(&v[c]));
      tmem_st_wait();
      // the words are in TMEM: the ring slot may be refilled (async proxy)
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&sf_empty[slot]));
        mbar_arrive_cluster(tsf_ready_leader0 + 8 * b);
      }
    }
  }

  tc_fence_before();
  cluster_sync();  // no CTA leaves while its peer may still signal it or read its TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

}  // namespace w4a4
