// gemm_tc2.cuh -- the FLCE GEMM on CTA pairs: tcgen05.mma.cta_group::2 with
// 256 x 256 output tiles split over two SMs (a cluster of two CTAs).
//
// Each CTA of the pair loads its own 128 rows of A and its own 128 rows (N)
// of B per pipeline stage of KS 64-column K slices (KS = 2: 128-deep stages
// of 64 KB, three of them), so each SM pulls two thirds of the bytes the
// single-CTA 128 x 256 tile needs per FLOP.  The leader CTA (rank 0) owns the
// pipeline:
//   * both producers' TMA loads count their bytes on the leader's `full`
//     barrier, which only the leader arms (with both CTAs' bytes);
//   * the leader's single MMA thread issues M=256, N=256, K=16 MMAs that read
//     A and B from both CTAs' shared memory and write each CTA's 128 rows of
//     the fp32 accumulator into that CTA's TMEM (two accumulators, so one
//     tile's epilogue overlaps the next tile's MMAs);
//   * its commits arrive on the `empty` and accumulator-full barriers of both
//     CTAs;
//   * every epilogue thread of both CTAs arrives on the leader's
//     accumulator-empty barrier.
// The epilogues are the single-CTA ones of gemm_tc.cuh: every CTA drains 128
// rows x 256 columns of its own TMEM, with four or eight warps.  Waits are
// bounded as there; the pair meets at a cluster barrier before freeing TMEM,
// so neither CTA leaves while the other may still touch its shared memory.
#pragma once

#include "gemm_tc.cuh"

namespace flce {

#ifndef FLCE_LOOP_FENCE
#define FLCE_LOOP_FENCE 1
#endif

constexpr int kPairBM = 256;  // rows of a pair tile (128 per CTA)
constexpr int kPairBN = 256;

// A stage holds KS slices of 64 K-columns (one 128-byte swizzle atom each).
template <int STAGES, int KS = 1>
struct Tc2Smem {
  static constexpr uint32_t kSliceBytes = 128 * kBK * 2;  // 128 rows x 64 K of one operand
  static constexpr uint32_t kABytes = KS * kSliceBytes;   // this CTA's 128 rows of A
  static constexpr uint32_t kBBytes = KS * kSliceBytes;   // this CTA's 128 rows (N) of B
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  // Output staging for TMA stores: 32 KB shared by the epilogue warps (two
  // 4 KB buffers each with four warps, one with eight).
  static constexpr uint32_t kOutStageBytes = 8 * 4096;
  static constexpr uint32_t kBarrierBytes = 256;
  static constexpr uint32_t kTotal =
      STAGES * kStageBytes + kOutStageBytes + kBarrierBytes + 1024;
  static constexpr uint32_t kTmemCols = 512;  // two 256-column fp32 accumulators
};

// Producer warp, MMA warp and EW epilogue warps.  With EW = 4 each warp
// drains its TMEM lane quarter's 32 rows x 256 columns; with EW = 8 two warps
// share a quarter, each draining 128 of the 256 columns, which gives every
// SM sub-partition a second warp to issue from while the first waits on
// TMEM, the SFU or memory.
constexpr int tc2_threads(int ew) { return 64 + 32 * ew; }

template <bool A_MN, bool B_MN, int MODE, int STAGES, int KS, int EW>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(tc2_threads(EW), 1)
    tc2_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, const TcShape sh,
                    const TcEpi ep) {
  using L = Tc2Smem<STAGES, KS>;
  const int k_stages = (sh.k_blocks + KS - 1) / KS;  // K past the tensors reads as zeros
  // Work units: (K split, tile); split s covers stages [s*kps, min((s+1)*kps, k_stages)).
  const int n_units = sh.num_tiles * sh.k_splits;
  const int kps = (k_stages + sh.k_splits - 1) / sh.k_splits;
  constexpr int BN = kPairBN;
  constexpr uint32_t kIdesc = make_idesc_bf16(kPairBM, kPairBN, A_MN, B_MN);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* out_stage = smem + STAGES * L::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(out_stage + L::kOutStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = int(blockIdx.x >> 1);
  const int n_pairs = int(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * 32 * EW);  // every epilogue thread of both CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = (*reinterpret_cast<volatile int*>(ep.status) != 0) ? 2 : 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (MODE != EPI_LSE && MODE != EPI_LSE_CAP) tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, L::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // A recomputation with no row group flagged has no work units; both CTAs
  // of the pair read the same flags and agree.
  const bool skip = *abort_flag != 0 || !any_group_flagged(ep);
  const uint64_t limit = ep.wait_limit_ns;

  if (!skip && warp == 0 && lane == 0) {
    // ------------------------------ producer ------------------------------
    const uint64_t pol = policy_evict_normal();
    uint32_t s = 0, ph = 0;
    uint32_t armed = 0;
    uint32_t armed_ph[STAGES];
#pragma unroll
    for (int i = 0; i < STAGES; ++i) armed_ph[i] = 0;
    bool ok = true;
    for (int u = pair; ok && u < n_units; u += n_pairs) {
      const int split = u / sh.num_tiles;
      int mt, nt;
      tile_coords(sh, u - split * sh.num_tiles, mt, nt);
      if (!tile_wanted(ep, sh, mt * kPairBM, kPairBM)) continue;
      const int m0 = mt * kPairBM + 128 * int(rank) + sh.a_mn_off;
      const int n0 = nt * kPairBN + 128 * int(rank) + sh.b_mn_off;
      const int kb1 = min(k_stages, (split + 1) * kps);
      for (int kb = split * kps; kb < kb1; ++kb) {
        if (!mbar_wait_bounded(&empty[s], ph ^ 1u, limit, abort_flag)) {
          record_timeout(ep, abort_flag);
          ok = false;
          break;
        }
        uint8_t* sa = smem + s * L::kStageBytes;
        uint8_t* sb = sa + L::kABytes;
        if (leader) {
          mbar_arrive_expect_tx(&full[s], 2 * L::kStageBytes);
          armed |= 1u << s;
          armed_ph[s] = ph;
        }
        const uint32_t bar = mapa_shared(&full[s], 0);
#pragma unroll
        for (int j = 0; j < KS; ++j) {
          uint8_t* saj = sa + j * L::kSliceBytes;
          uint8_t* sbj = sb + j * L::kSliceBytes;
          const int ka = (kb * KS + j) * kBK + sh.a_k_off;
          const int kbb = (kb * KS + j) * kBK + sh.b_k_off;
          if (!A_MN) {
            tma_load_2d_pair(saj, &tmA, bar, ka, m0, pol);
          } else {
            tma_load_2d_pair(saj, &tmA, bar, m0, ka, pol);
            tma_load_2d_pair(saj + 8192, &tmA, bar, m0 + 64, ka, pol);
          }
          if (!B_MN) {
            tma_load_2d_pair(sbj, &tmB, bar, kbb, n0, pol);
          } else {
            tma_load_2d_pair(sbj, &tmB, bar, n0, kbb, pol);
            tma_load_2d_pair(sbj + 8192, &tmB, bar, n0 + 64, kbb, pol);
          }
        }
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    if (leader && (!ok || *abort_flag)) {
      for (int i = 0; i < STAGES; ++i)
        if (armed & (1u << i)) mbar_wait_bounded(&full[i], armed_ph[i], kDrainLimitNs, nullptr);
    }
  } else if (!skip && leader && warp == 1 && lane == 0) {
    // --------------------------- MMA issuer (leader) -----------------------
    uint32_t s = 0, ph = 0, acc = 0, aph = 0;
    bool ok = true;
    for (int u = pair; ok && u < n_units; u += n_pairs) {
      const int split = u / sh.num_tiles;
      {
        int mt, nt;
        tile_coords(sh, u - split * sh.num_tiles, mt, nt);
        if (!tile_wanted(ep, sh, mt * kPairBM, kPairBM)) continue;
      }
      if (!mbar_wait_bounded(&tempty[acc], aph ^ 1u, limit, abort_flag)) {
        record_timeout(ep, abort_flag);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d = tmem_base + acc * BN;
      const int kb0 = split * kps;
      const int kb1 = min(k_stages, kb0 + kps);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait_bounded(&full[s], ph, limit, abort_flag)) {
          record_timeout(ep, abort_flag);
          ok = false;
          break;
        }
#if FLCE_LOOP_FENCE
        tc_fence_after();
#endif
        const uint32_t a_addr = smem_u32(smem + s * L::kStageBytes);
        const uint32_t b_addr = a_addr + L::kABytes;
#pragma unroll
        for (int j = 0; j < KS; ++j) {
          const uint32_t aj = a_addr + j * L::kSliceBytes;
          const uint32_t bj = b_addr + j * L::kSliceBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = A_MN ? make_sdesc_sw128(aj + kk * 2048, 8192, 1024)
                                     : make_sdesc_sw128(aj + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? make_sdesc_sw128(bj + kk * 2048, 8192, 1024)
                                     : make_sdesc_sw128(bj + kk * 32, 16, 1024);
            umma_bf16_pair(d, ad, bd, kIdesc, ((kb - kb0) | j | kk) != 0 ? 1u : 0u);
          }
        }
        umma_commit_pair(mapa_shared(&empty[s], 0));
        umma_commit_pair(mapa_shared(&empty[s], 1));
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) break;
      umma_commit_pair(mapa_shared(&tfull[acc], 0));
      umma_commit_pair(mapa_shared(&tfull[acc], 1));
      acc ^= 1u;
      if (acc == 0) aph ^= 1u;
    }
    umma_commit_pair(mapa_shared(drain, 0));
    mbar_wait_bounded(drain, 0, kDrainLimitNs, nullptr);
  } else if (!skip && warp >= 2) {
    // ------------------------------- epilogue ------------------------------
    static_assert(EW == 4 || EW == 8, "four or eight epilogue warps");
    constexpr int kChunks = (BN / 32) * 4 / EW;  // 32-column chunks per warp
    const int q = warp & 3;                      // TMEM lane quarter this warp may read
    const int half = (warp - 2) >> 2;            // 0, or 1 for the second warp of a quarter
    const int c_lo = half * kChunks, c_hi = c_lo + kChunks;
    const int r = q * 32 + lane;
    uint32_t acc = 0, aph = 0;
    uint32_t pieces = 0;  // bf16 output pieces this warp has stored by TMA
    uint8_t* my_stage = out_stage + (warp - 2) * (L::kOutStageBytes / EW);
    for (int u = pair; u < n_units; u += n_pairs) {
      const int split = u / sh.num_tiles;
      int mt, nt;
      tile_coords(sh, u - split * sh.num_tiles, mt, nt);
      if (!tile_wanted(ep, sh, mt * kPairBM, kPairBM)) continue;
      constexpr bool kQ = MODE == EPI_LSE_Q || MODE == EPI_LSE_Q_CAP;
      const int64_t lab_pre =
          kQ ? epi_row_label(ep, sh, mt * kPairBM + 128 * int(rank), q * 32 + lane) : 0;
      const bool got = mbar_wait_bounded(&tfull[acc], aph, limit, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) record_timeout(ep, abort_flag);
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (uint32_t(q * 32) << 16) + acc * BN;
      const int m0 = mt * kPairBM + 128 * int(rank);
      const int n0 = nt * kPairBN;
      TmaSink sink{&tmC, my_stage, lane, n0, ep.out_row_off + m0 + q * 32, &pieces,
                   ep.out_cols, ep.out_row_off + sh.M, 8 / EW};
      // LSE partial slice: one per 256 columns with four warps, per 128 with eight.
      const int part = EW == 8 ? 2 * nt + half : nt;
      if (MODE == EPI_LSE) epi_lse<BN, false>(ep, sh, m0, n0, part, r, taddr, c_lo, c_hi);
      if (MODE == EPI_LSE_CAP) epi_lse<BN, true>(ep, sh, m0, n0, part, r, taddr, c_lo, c_hi);
      if (MODE == EPI_GRAD)
        epi_grad<BN, false>(ep, sh, m0, n0, r, taddr, &sink, c_lo, c_hi);
      if (MODE == EPI_GRAD_CAP)
        epi_grad<BN, true>(ep, sh, m0, n0, r, taddr, &sink, c_lo, c_hi);
      // Ten warps leave each thread 200 registers: 64-column TMEM loads.
      if (MODE == EPI_DX)
        epi_dx<BN, EW == 8 ? 64 : 128>(ep, sh, m0, n0, r, taddr, split, &sink, c_lo, c_hi);
      if (MODE == EPI_DW) epi_dw<BN>(ep, sh, m0, n0, r, taddr, &sink, c_lo, c_hi);
      if (MODE == EPI_LSE_Q)
        epi_lse_q<BN, false, kChunks>(ep, sh, m0, n0, part, r, taddr, &sink, c_lo, c_hi,
                                      lab_pre);
      if (MODE == EPI_LSE_Q_CAP)
        epi_lse_q<BN, true, kChunks>(ep, sh, m0, n0, part, r, taddr, &sink, c_lo, c_hi,
                                     lab_pre);
      tc_fence_before();
      mbar_arrive_cluster(mapa_shared(&tempty[acc], 0));
      acc ^= 1u;
      if (acc == 0) aph ^= 1u;
    }
    // Output stores still reading the staging buffers finish before exit.
    if (lane == 0) bulk_wait_group<0>();
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();  // the pair leaves together: no CTA exits while its peer may read it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, L::kTmemCols);
  }
}

}  // namespace flce
