// The W4A4 GEMM on CTA pairs: one tcgen05 MMA (cta_group::2) spans the two
// SMs of a cluster of 2, computing a 256 x NB tile (NB = 256 or 384) of
//   Y = bf16( deq(Qx) deq(Qr)^T  +  T L2t^T )
// (devpress.csdn.net SVDQuant walkthrough, eq. (2), eq. (5) and Fig. 6).
// Each CTA of the pair stages its own 128 rows of the A operand (Qx, then T)
// and its own NB/2 rows of the B operand (Qr, then L2t); each CTA also stages
// the A scales of its rows and the B scales of all NB columns, and its scale
// warps write them into its own TMEM (the pair MMA reads both).
//
// NB = 384 (two MMAs per K block: N = 256 into accumulator columns [0, 256),
// N = 128 into [256, 384)) reads 16 % fewer operand bytes per FLOP than
// NB = 256; its accumulator leaves room in TMEM for two scale buffers only,
// used in turn (buffer it % 2 is free once the commit of item it - 2 landed).
// With NB = 256 every ring stage has its own scale buffer.
//
// Persistent: cluster c walks pair tiles c, c + clusters, ... Each tile is a
// sequence of items (K/256 FP4 k-tiles, then ceil(r/64) low-rank k-tiles).
// Roles per CTA (448 threads), identical in both CTAs except where noted:
//   warps 0-7   epilogue: drain this CTA's 128 x NB fp32 accumulator,
//               release it to the even CTA's MMA issuer, write Y through
//               128B-swizzled boxes and TMA stores
//   warp 8      producer: TMA loads of this CTA's item rows and scale atoms,
//               counted on this CTA's own stage barrier
//   warp 9      TMEM allocation (both CTAs); in the even CTA one lane issues
//               the pair MMAs of each item once both CTAs' scale warps have
//               reported it, and releases each ring stage (with its TMEM
//               scale buffer) and the accumulator of both CTAs with
//               multicast tcgen05.commit
//   warps 10-13 scale warps: wait for this CTA's stage, put its scales in a
//               TMEM scale buffer (tcgen05.st), report to the even CTA
// Every wait is bounded; on a timeout the kernel records a device error word,
// every role stops, and both CTAs still meet at the final cluster barrier.
#pragma once

#include <cuda_bf16.h>

#include "svdq_gemm_common.cuh"
#include "svdq_gemm_qnext.cuh"
#include "svdq_ptx.cuh"

namespace svdq {

constexpr int kPairBM = 256;                          // M rows per pair tile (128 per CTA)
constexpr int kPairStageA = 128 * kGemmBKBytes;       // 16 KB: this CTA's 128 Qx rows (or T rows)
constexpr int kPairStageSfa = kGemmKBPerStage * kSfAtomBytes;       // 2 KB

template <int NB>
struct PairCfg {
  static_assert(NB == 256 || NB == 384, "pair tile width");
  static constexpr int kBRows = NB / 2;                               // B rows per CTA
  static constexpr int kStageB = kBRows * kGemmBKBytes;               // 16 | 24 KB
  static constexpr int kSfbBlocks = NB / 128;                         // 128-row blocks of B scales
  static constexpr int kStageSfb = kSfbBlocks * kGemmKBPerStage * kSfAtomBytes;   // 4 | 6 KB
  static constexpr int kStageBytes = kPairStageA + kStageB + kPairStageSfa + kStageSfb;   // 38 | 48 KB
  static constexpr int kStages = NB == 256 ? 5 : 4;
  static constexpr uint32_t kSfCols = 4 * kGemmKBPerStage * (1 + kSfbBlocks);   // 48 | 64 TMEM columns
  static constexpr int kSfBufs = (int)((kTmemCols - NB) / kSfCols);             // 5 | 2
  static constexpr bool kSfPerStage = kSfBufs >= kStages;
  static_assert(kSfBufs >= 2, "scale buffers");
  static constexpr int kEpiOffset = kStages * kStageBytes;
  static constexpr int kBarOffset = kEpiOffset + kGemmEpiWarps * kEpiBoxBytes;
  static constexpr int kBytes = kBarOffset + 512 + 1024;
  // TMEM column of the scale buffer of item `it` in ring stage `s`
  __device__ static uint32_t sf_col(uint32_t it, int s) {
    return (uint32_t)NB + (kSfPerStage ? (uint32_t)s : it % (uint32_t)kSfBufs) * kSfCols;
  }
};

// Launched with a cluster dimension of (2, 1, 1).
// tm_qr / tm_l2 boxes are 128 rows (NB = 256) or 64 rows (NB = 384).
// tm_sfa / tm_sfb view a native scale buffer as 3-D uint8
// [row blocks][K/64 * 2 chunks][256 bytes]; box {256, 8, 1 | NB/128} (4 atoms per row block).
// QNEXT: the epilogue also quantizes Y for the next layer (svdq_gemm_qnext.cuh),
// and stores Y itself only when store_y is set.
template <int NB, bool QNEXT = false>
__global__ void __launch_bounds__(kGemmThreads, 1) svdq_gemm_pair_kernel(
    const __grid_constant__ CUtensorMap tm_qx, const __grid_constant__ CUtensorMap tm_qr,
    const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
    const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_l2,
    const __grid_constant__ CUtensorMap tm_y, int M, int N, int K, int rank, NextQuant nq, int store_y) {
  static_assert(!QNEXT || NB == 256, "the next layer's quantization runs on 256 x 256 tiles");
  using C = PairCfg<NB>;
  constexpr int STAGES = C::kStages;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
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
  const int tiles_n = N / NB;
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
  __shared__ float2 rcp_tbl[QNEXT ? 128 : 1];   // bracket of 1/s per E4M3 byte with the sign bit clear
  if (QNEXT && threadIdx.x < 128) rcp_tbl[threadIdx.x] = e4m3_recip_bracket(threadIdx.x);
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
  grid_dependency_wait();     // the previous kernel's outputs (Qx, Sx, T) are complete
  grid_launch_dependents();

  if (warp == kProducerWarp) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer (both CTAs)
      uint32_t it = 0;
      bool ok = true;
      for (int tile = cluster; tile < ntiles && ok; tile += nclusters) {
        const int m0 = (tile / tiles_n) * kPairBM + 128 * (int)crank;   // this CTA's A rows
        const int n0 = (tile % tiles_n) * NB;                           // the pair's N columns
        for (int kt = 0; kt < n_fp4_kt + n_lr_kt; ++kt, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(empty + s, ((it / STAGES) & 1u) ^ 1u, kDevErrTimeoutEmpty)) {
            ok = false;
            break;
          }
          unsigned char* sa = smem + s * C::kStageBytes;
          unsigned char* sb = sa + kPairStageA;
          if (kt < n_fp4_kt) {
            unsigned char* sfa = sb + C::kStageB;
            unsigned char* sfb = sfa + kPairStageSfa;
            mbar_arrive_expect_tx(full + s, (uint32_t)C::kStageBytes);
            tma_load_2d(sa, &tm_qx, full + s, kt * kGemmBKBytes, m0);
            if (NB == 256) {
              tma_load_2d(sb, &tm_qr, full + s, kt * kGemmBKBytes, n0 + 128 * (int)crank);
            } else {   // rows n0 + 128 c + [0, 128) for the first MMA, n0 + 256 + 64 c + [0, 64) for the second
              tma_load_2d(sb, &tm_qr, full + s, kt * kGemmBKBytes, n0 + 128 * (int)crank);
              tma_load_2d(sb + 64 * kGemmBKBytes, &tm_qr, full + s, kt * kGemmBKBytes, n0 + 128 * (int)crank + 64);
              tma_load_2d(sb + 128 * kGemmBKBytes, &tm_qr, full + s, kt * kGemmBKBytes, n0 + 256 + 64 * (int)crank);
            }
            tma_load_3d(sfa, &tm_sfa, full + s, 0, kt * kGemmKBPerStage * 2, m0 >> 7);
            tma_load_3d(sfb, &tm_sfb, full + s, 0, kt * kGemmKBPerStage * 2, n0 >> 7);
          } else {
            const int c = kt - n_fp4_kt;
            mbar_arrive_expect_tx(full + s, (uint32_t)(kPairStageA + C::kStageB));
            tma_load_2d(sa, &tm_t, full + s, c * kGemmLrK, m0);
            if (NB == 256) {
              tma_load_2d(sb, &tm_l2, full + s, c * kGemmLrK, n0 + 128 * (int)crank);
            } else {
              tma_load_2d(sb, &tm_l2, full + s, c * kGemmLrK, n0 + 128 * (int)crank);
              tma_load_2d(sb + 64 * kGemmBKBytes, &tm_l2, full + s, c * kGemmLrK, n0 + 128 * (int)crank + 64);
              tma_load_2d(sb + 128 * kGemmBKBytes, &tm_l2, full + s, c * kGemmLrK, n0 + 256 + 64 * (int)crank);
            }
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
        // stage s has landed
        if (!mbar_wait(full + s, (it / STAGES) & 1u, kDevErrTimeoutFull)) {
          ok = false;
          break;
        }
        // its scale buffer is free: with one buffer per stage, the commit that
        // released the stage's previous use (which preceded this refill) freed
        // it; with buffers used in turn, wait for the commit of the buffer's
        // previous item (items complete in order, so that phase of its stage's
        // barrier is the latest one that can have completed)
        if (!C::kSfPerStage && it >= (uint32_t)C::kSfBufs) {
          const uint32_t pj = it - (uint32_t)C::kSfBufs;
          if (!mbar_wait(empty + pj % STAGES, (pj / STAGES) & 1u, kDevErrTimeoutScales)) {
            ok = false;
            break;
          }
        }
        tc_fence_after();
        if (kt < n_fp4_kt) {
          const unsigned char* sfa = smem + s * C::kStageBytes + kPairStageA + C::kStageB;
          const unsigned char* sfb = sfa + kPairStageSfa;
          scales_to_tmem(tmem, q, lane, sfa, sfb, sfb + 4 * kSfAtomBytes, C::sf_col(it, s),
                         NB == 384 ? sfb + 8 * kSfAtomBytes : nullptr);
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
      // The issuing thread runs only a few MMAs ahead of the tensor pipe, so
      // every cycle it spends between two items' MMAs can leave the pipe idle.
      // The loop is kept short: the stage index and barrier parity are carried
      // from item to item, the shared-memory descriptors are offsets of two
      // precomputed ones, and whether the next item's scales are in place is
      // tested before this item's MMAs are queued, so that in the common case
      // no barrier wait stands between two items.
      uint32_t tcount = 0;
      bool ok = true;
      const uint32_t idesc = idesc_nvfp4(kPairBM, 256);
      const uint32_t idesc2 = idesc_nvfp4(kPairBM, 128);
      const uint32_t idesc_lr = idesc_bf16(kPairBM, 256);
      const uint32_t idesc_lr2 = idesc_bf16(kPairBM, 128);
      // descriptors of stage 0; a stage, a 64-element K block (32 bytes) and
      // the B rows of the second MMA are offsets of the 16-byte address field
      // (shared addresses stay below 2^18, so the field cannot carry over)
      const uint64_t dA0 = smem_desc(smem_u32(smem), 16, 1024, kSwizzle128B);
      const uint64_t dB0 = smem_desc(smem_u32(smem) + kPairStageA, 16, 1024, kSwizzle128B);
      constexpr uint32_t kStageDesc = (uint32_t)C::kStageBytes >> 4;
      constexpr uint32_t kB2Desc = (128u * kGemmBKBytes) >> 4;
      constexpr uint32_t kKbDesc = 32u >> 4;
      const int n_items = n_fp4_kt + n_lr_kt;
      int s = 0;                 // ring stage and barrier parity of the current item
      uint32_t ph = 0;
      uint32_t sfbuf = 0;        // item index mod 2 (scale buffers used in turn)
      bool ready = false;        // the current item's stage and scales are known to be in place
      for (int tile = cluster; tile < ntiles && ok; tile += nclusters, ++tcount) {
        // acc_empty and sf_ready count arrivals from both CTAs, each announcing
        // TMEM reads / writes that a tcgen05.wait already completed (see
        // mbar_arrive_remote); the waits take CTA-scope acquire and are
        // followed by tcgen05.fence::after_thread_sync before the MMAs
        if (!mbar_wait(acc_empty, (tcount & 1u) ^ 1u, kDevErrTimeoutAccum)) {
          ok = false;
          break;
        }
        for (int kt = 0; kt < n_items; ++kt) {
          // both CTAs' scale warps saw stage s full and put its scales in TMEM
          if (!ready && !mbar_wait(sf_ready + s, ph, kDevErrTimeoutScales)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int s1 = s + 1 == STAGES ? 0 : s + 1;
          const uint32_t ph1 = s + 1 == STAGES ? ph ^ 1u : ph;
          ready = mbar_test(sf_ready + s1, ph1);
          const uint64_t ad = dA0 + (uint64_t)((uint32_t)s * kStageDesc);
          const uint64_t bd = dB0 + (uint64_t)((uint32_t)s * kStageDesc);
          if (kt < n_fp4_kt) {
            const uint32_t sfa = tmem + (uint32_t)NB + (C::kSfPerStage ? (uint32_t)s : sfbuf) * C::kSfCols;
            const uint32_t sfb = sfa + 4 * kGemmKBPerStage;
            const uint32_t sfb2 = sfa + 12 * kGemmKBPerStage;
            const int kbs = min(kGemmKBPerStage, kb_total - kt * kGemmKBPerStage);
#pragma unroll
            for (int kb = 0; kb < kGemmKBPerStage; ++kb) {
              if (kb < kbs) {
                const uint32_t acc = (kt | kb) != 0 ? 1u : 0u;
                mma_nvfp4_pair(tmem, ad + kb * kKbDesc, bd + kb * kKbDesc, idesc, sfa + 4 * kb, sfb + 8 * kb, acc);
                if (NB == 384)
                  mma_nvfp4_pair(tmem + 256, ad + kb * kKbDesc, bd + kB2Desc + kb * kKbDesc, idesc2, sfa + 4 * kb,
                                 sfb2 + 4 * kb, acc);
              }
            }
          } else {
            const int k16 = min(kGemmLrK, rank - (kt - n_fp4_kt) * kGemmLrK) / 16;
#pragma unroll
            for (int j = 0; j < kGemmLrK / 16; ++j) {
              if (j < k16) {
                mma_bf16_pair(tmem, ad + j * kKbDesc, bd + j * kKbDesc, idesc_lr, 1u);
                if (NB == 384) mma_bf16_pair(tmem + 256, ad + j * kKbDesc, bd + kB2Desc + j * kKbDesc, idesc_lr2, 1u);
              }
            }
          }
          tc_commit_pair(empty + s, 0x3);     // stage s and its scale buffer, in both CTAs, are free
          sfbuf ^= 1u;
          s = s1;
          ph = ph1;
        }
        if (ok) tc_commit_pair(acc_full, 0x3);   // both halves of the tile's accumulator are complete
      }
      if (!ok) {
        tc_commit_pair(mma_drain, 0x1);
        mbar_wait(mma_drain, 0, kDevErrTimeoutAccum);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3, h = warp >> 2;
    unsigned char* box = smem + C::kEpiOffset + warp * kEpiBoxBytes;
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
    if (lane == 0 && (!QNEXT || store_y)) prefetch_tmap(&tm_y);
    uint32_t tcount = 0;
    for (int tile = cluster; tile < ntiles; tile += nclusters, ++tcount) {
      const int m0 = (tile / tiles_n) * kPairBM + 128 * (int)crank;
      const int n0 = (tile % tiles_n) * NB;
      const bool ok = mbar_wait(acc_full, tcount & 1u, kDevErrTimeoutAccum);
      tc_fence_after();
      if (!ok || device_error_set()) break;
      // warp (q, h): lanes 32q.., accumulator columns h * NB/2 + [0, NB/2)
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * (NB / 2));
      const bool store = m0 + 32 * q < M;
      uint32_t p[64];
      epilogue_drain_pack<4>(taddr, p);
      if (NB == 256) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(acc_empty_leader);   // this warp's part of the accumulator is drained
        if (QNEXT)
          epilogue_quantize_next<2>(p, box, nq, rcp_tbl, &tm_y, store_y != 0, m0 + 32 * q, n0 + h * 128, M, N, lane);
        else
          epilogue_store_band<2>(p, box, &tm_y, n0 + h * 128, m0 + 32 * q, lane, store);
      } else {   // drain all 192 columns before releasing the accumulator, then store
        uint32_t p2[32];
        epilogue_drain_pack<2>(taddr + 128, p2);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(acc_empty_leader);
        epilogue_store_band<2>(p, box, &tm_y, n0 + h * 192, m0 + 32 * q, lane, store);
        epilogue_store_band<1>(p2, box, &tm_y, n0 + h * 192 + 128, m0 + 32 * q, lane, store);
      }
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
