// The W4A4 GEMM on CTA pairs: one tcgen05 MMA (cta_group::2) spans the two
// SMs of a cluster of 2, computing a 256 x 256 tile of
//   Y = bf16( deq(Qx) deq(Qr)^T  +  T L2t^T )
// (devpress.csdn.net SVDQuant walkthrough, eq. (2), eq. (5) and Fig. 6).
// Each CTA of the pair stages its own 128 rows of the A operand (Qx, then T)
// and its own 128 rows of the B operand (Qr, then L2t), so a pair reads 2/3 of
// the operand bytes two independent 128 x 256 tiles would; each CTA also
// stages the A scales of its rows and the B scales of all 256 columns, and its
// scale warps write them into its own TMEM (the pair MMA reads both).
//
// Persistent: cluster c walks pair tiles c, c + clusters, ... Each tile is a
// sequence of items (K/256 FP4 k-tiles, then ceil(r/64) low-rank k-tiles).
// Roles per CTA (448 threads), identical in both CTAs except where noted:
//   warps 0-7   epilogue: drain this CTA's 128 x 256 fp32 accumulator,
//               release it to the even CTA's MMA issuer, write Y through
//               128B-swizzled boxes and TMA stores
//   warp 8      producer: TMA loads of this CTA's item rows and scale atoms,
//               counted on this CTA's own stage barrier
//   warp 9      TMEM allocation (both CTAs); in the even CTA one lane issues
//               the pair MMAs of each item once both CTAs' scale warps have
//               reported it, and releases each ring stage (with its TMEM
//               scale buffer) and the accumulator of both CTAs with
//               multicast tcgen05.commit
//   warps 10-13 scale warps: wait for this CTA's stage, put its scales in the
//               stage's TMEM scale buffer (tcgen05.st), report to the even CTA
// Every wait is bounded; on a timeout the kernel records a device error word,
// every role stops, and both CTAs still meet at the final cluster barrier.
#pragma once

#include <cuda_bf16.h>

#include "svdq_gemm_common.cuh"
#include "svdq_ptx.cuh"

namespace svdq {

constexpr int kPairBM = 256;                          // M rows per pair tile (128 per CTA)
constexpr int kPairBN = 256;                          // N columns per pair tile (B rows: 128 per CTA)
constexpr int kPairStageA = 128 * kGemmBKBytes;       // 16 KB: this CTA's 128 Qx rows (or T rows)
constexpr int kPairStageB = 128 * kGemmBKBytes;       // 16 KB: this CTA's 128 Qr rows (or L2t rows)
constexpr int kPairStageSfa = kGemmKBPerStage * kSfAtomBytes;       // 2 KB
constexpr int kPairStageSfb = 2 * kGemmKBPerStage * kSfAtomBytes;   // 4 KB (both 128-row halves of N)
constexpr int kPairStageBytes = kPairStageA + kPairStageB + kPairStageSfa + kPairStageSfb;   // 38 KB

template <int STAGES>
struct PairSmem {
  static constexpr int kEpiOffset = STAGES * kPairStageBytes;
  static constexpr int kBarOffset = kEpiOffset + kGemmEpiWarps * kEpiBoxBytes;
  static constexpr int kBytes = kBarOffset + 512 + 1024;
};

// Launched with a cluster dimension of (2, 1, 1).
// tm_sfa / tm_sfb view a native scale buffer as 3-D uint8
// [row blocks][K/64 * 2 chunks][256 bytes]; box {256, 8, 1|2} (4 atoms per row block).
template <int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1) svdq_gemm_pair_kernel(
    const __grid_constant__ CUtensorMap tm_qx, const __grid_constant__ CUtensorMap tm_qr,
    const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
    const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_l2,
    const __grid_constant__ CUtensorMap tm_y, int M, int N, int K, int rank) {
  using L = PairSmem<STAGES>;
  static_assert(STAGES <= kMaxSfBufs, "one TMEM scale buffer per ring stage");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOffset);
  uint64_t* empty = full + STAGES;
  uint64_t* sf_ready = empty + STAGES;      // even CTA: both CTAs' scale warps report here
  uint64_t* acc_full = sf_ready + STAGES;
  uint64_t* acc_empty = acc_full + 1;       // even CTA: both CTAs' epilogue warps report here
  uint64_t* mma_drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const bool leader = crank == 0;
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  const int tiles_n = N / kPairBN;
  const int ntiles = ((M + kPairBM - 1) / kPairBM) * tiles_n;
  const int kb_total = K >> 6;
  const int n_fp4_kt = (kb_total + kGemmKBPerStage - 1) / kGemmKBPerStage;
  const int n_lr_kt = (rank + kGemmLrK - 1) / kGemmLrK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < STAGES; ++b) mbar_init(sf_ready + b, 2 * kSfWarps);
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * kGemmEpiWarps);
    mbar_init(mma_drain, 1);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&tm_qx);
    prefetch_tmap(&tm_qr);
    prefetch_tmap(&tm_sfa);
    prefetch_tmap(&tm_sfb);
    if (rank > 0) {
      prefetch_tmap(&tm_t);
      prefetch_tmap(&tm_l2);
    }
  }
  tc_fence_before();
  cluster_sync();   // barriers of both CTAs initialised, TMEM allocated in both
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer (both CTAs)
      uint32_t it = 0;
      bool ok = true;
      for (int tile = cluster; tile < ntiles && ok; tile += nclusters) {
        const int m0 = (tile / tiles_n) * kPairBM + 128 * (int)crank;   // this CTA's A rows
        const int n0 = (tile % tiles_n) * kPairBN;                      // the pair's N columns
        for (int kt = 0; kt < n_fp4_kt + n_lr_kt; ++kt, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(empty + s, ((it / STAGES) & 1u) ^ 1u, kDevErrTimeoutEmpty)) {
            ok = false;
            break;
          }
          unsigned char* sa = smem + s * kPairStageBytes;
          unsigned char* sb = sa + kPairStageA;
          if (kt < n_fp4_kt) {
            unsigned char* sfa = sb + kPairStageB;
            unsigned char* sfb = sfa + kPairStageSfa;
            mbar_arrive_expect_tx(full + s, (uint32_t)kPairStageBytes);
            tma_load_2d(sa, &tm_qx, full + s, kt * kGemmBKBytes, m0);
            tma_load_2d(sb, &tm_qr, full + s, kt * kGemmBKBytes, n0 + 128 * (int)crank);
            tma_load_3d(sfa, &tm_sfa, full + s, 0, kt * kGemmKBPerStage * 2, m0 >> 7);
            tma_load_3d(sfb, &tm_sfb, full + s, 0, kt * kGemmKBPerStage * 2, n0 >> 7);
          } else {
            const int c = kt - n_fp4_kt;
            mbar_arrive_expect_tx(full + s, (uint32_t)(kPairStageA + kPairStageB));
            tma_load_2d(sa, &tm_t, full + s, c * kGemmLrK, m0);
            tma_load_2d(sb, &tm_l2, full + s, c * kGemmLrK, n0 + 128 * (int)crank);
          }
        }
      }
      if (device_error_set()) {
        for (uint32_t j = it > (uint32_t)STAGES ? it - STAGES : 0u; j < it; ++j)
          mbar_wait(full + j % STAGES, (j / STAGES) & 1u, kDevErrTimeoutFull);
      }
    }
  } else if (warp >= kSfWarp0) {
    // ------------------------------------------------------------------ scale warps (both CTAs)
    const int q = warp & 3;
    const uint32_t sf_ready_leader = mapa_shared(smem_u32(sf_ready), 0);
    uint32_t it = 0;
    bool ok = true;
    for (int tile = cluster; tile < ntiles && ok; tile += nclusters) {
      for (int kt = 0; kt < n_fp4_kt + n_lr_kt; ++kt, ++it) {
        const int s = it % STAGES;
        // stage s has landed; its scale buffer was freed by the commit that
        // released the stage's previous use (which preceded this refill)
        if (!mbar_wait(full + s, (it / STAGES) & 1u, kDevErrTimeoutFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (kt < n_fp4_kt) {
          const unsigned char* sfa = smem + s * kPairStageBytes + kPairStageA + kPairStageB;
          const unsigned char* sfb = sfa + kPairStageSfa;
          scales_to_tmem(tmem, q, lane, sfa, sfb, sfb + kPairStageSfb / 2, sf_buf_col(s));
          tmem_st_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(sf_ready_leader + 8u * (uint32_t)s);   // this CTA's stage + scales ready
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0 && leader) {
      // ---------------------------------------------------------------- MMA issuer (even CTA)
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      const uint32_t idesc = idesc_nvfp4(kPairBM, kPairBN);
      const uint32_t idesc_lr = idesc_bf16(kPairBM, kPairBN);
      for (int tile = cluster; tile < ntiles && ok; tile += nclusters, ++tcount) {
        if (!mbar_wait_cluster(acc_empty, (tcount & 1u) ^ 1u, kDevErrTimeoutAccum)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kt = 0; kt < n_fp4_kt + n_lr_kt; ++kt, ++it) {
          const int s = it % STAGES;
          // both CTAs' scale warps saw stage s full and put its scales in TMEM
          if (!mbar_wait_cluster(sf_ready + s, (it / STAGES) & 1u, kDevErrTimeoutScales)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * kPairStageBytes);
          const uint32_t sb = sa + kPairStageA;
          if (kt < n_fp4_kt) {
            const uint32_t sfa = tmem + sf_buf_col(s);
            const uint32_t sfb = sfa + 4 * kGemmKBPerStage;
            const int kbs = min(kGemmKBPerStage, kb_total - kt * kGemmKBPerStage);
            for (int kb = 0; kb < kbs; ++kb) {
              const uint64_t ad = smem_desc(sa + kb * 32, 16, 1024, kSwizzle128B);
              const uint64_t bd = smem_desc(sb + kb * 32, 16, 1024, kSwizzle128B);
              mma_nvfp4_pair(tmem, ad, bd, idesc, sfa + 4 * kb, sfb + 8 * kb, (kt | kb) != 0 ? 1u : 0u);
            }
          } else {
            const int c = kt - n_fp4_kt;
            const int k16 = min(kGemmLrK, rank - c * kGemmLrK) / 16;
            for (int j = 0; j < k16; ++j) {
              const uint64_t ad = smem_desc(sa + j * 32, 16, 1024, kSwizzle128B);
              const uint64_t bd = smem_desc(sb + j * 32, 16, 1024, kSwizzle128B);
              mma_bf16_pair(tmem, ad, bd, idesc_lr, 1u);
            }
          }
          tc_commit_pair(empty + s, 0x3);     // stage s and its scale buffer, in both CTAs, are free
        }
        tc_commit_pair(acc_full, 0x3);        // both halves of the tile's accumulator are complete
      }
      if (!ok) {
        tc_commit_pair(mma_drain, 0x1);
        mbar_wait(mma_drain, 0, kDevErrTimeoutAccum);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3, h = warp >> 2;
    unsigned char* box = smem + L::kEpiOffset + warp * kEpiBoxBytes;
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
    if (lane == 0) prefetch_tmap(&tm_y);
    uint32_t tcount = 0;
    for (int tile = cluster; tile < ntiles; tile += nclusters, ++tcount) {
      const int m0 = (tile / tiles_n) * kPairBM + 128 * (int)crank;
      const int n0 = (tile % tiles_n) * kPairBN;
      const bool ok = mbar_wait(acc_full, tcount & 1u, kDevErrTimeoutAccum);
      tc_fence_after();
      if (!ok || device_error_set()) break;
      uint32_t p[64];
      epilogue_drain_pack(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * 128), p);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(acc_empty_leader);   // this warp's part of the accumulator is drained
      epilogue_store_band(p, box, &tm_y, n0 + h * 128, m0 + 32 * q, lane, m0 + 32 * q < M);
    }
    if (lane == 0) bulk_wait<0>();
  }

  tc_fence_before();
  cluster_sync();   // no CTA leaves while its peer may still signal its barriers
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace svdq
