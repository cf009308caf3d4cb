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

// QLR: the epilogue also forms the next layer's down-projection (next rank 16
// or 32): a ring of 4 stages (so that TMEM keeps 32 columns for T' and shared
// memory two staging boxes per epilogue warp and the tile's L1p' slice).
template <int NB, bool QLR = false>
struct PairCfg {
  static_assert(NB == 256 || NB == 384, "pair tile width");
  static_assert(!QLR || NB == 256, "the next layer's down-projection runs on 256 x 256 tiles");
  static constexpr int kBRows = NB / 2;                               // B rows per CTA
  static constexpr int kStageB = kBRows * kGemmBKBytes;               // 16 | 24 KB
  static constexpr int kSfbBlocks = NB / 128;                         // 128-row blocks of B scales
  static constexpr int kStageSfb = kSfbBlocks * kGemmKBPerStage * kSfAtomBytes;   // 4 | 6 KB
  static constexpr int kStageBytes = kPairStageA + kStageB + kPairStageSfa + kStageSfb;   // 38 | 48 KB
  static constexpr int kStages = QLR ? 4 : NB == 256 ? 5 : 4;
  static constexpr uint32_t kSfCols = 4 * kGemmKBPerStage * (1 + kSfbBlocks);   // 48 | 64 TMEM columns
  static constexpr uint32_t kTpCols = QLR ? 32 : 0;                             // T' accumulator columns
  static constexpr int kSfBufs = (int)((kTmemCols - NB - kTpCols) / kSfCols);   // 5 | 2 (4 with QLR)
  static constexpr uint32_t kTpCol = kTmemCols - kTpCols;                       // T' at columns [480, 512)
  static constexpr bool kSfPerStage = kSfBufs >= kStages;
  static_assert(kSfBufs >= 2, "scale buffers");
  static_assert(NB + kSfBufs * kSfCols <= kTpCol, "TMEM plan");
  static constexpr int kEpiBoxes = QLR ? 2 : 1;                                 // staging boxes per epilogue warp
  static constexpr int kEpiOffset = kStages * kStageBytes;
  static constexpr int kL1Half = 2 * 16 * 128;   // L1p' columns of one tile half: 2 boxes of <= 16 rows x 64
  static constexpr int kL1Offset = kEpiOffset + kGemmEpiWarps * kEpiBoxes * kEpiBoxBytes;
  static constexpr int kBarOffset = kL1Offset + (QLR ? 2 * kL1Half : 0);
  static constexpr int kBytes = kBarOffset + 512 + 1024;
  // TMEM column of the scale buffer of item `it` in ring stage `s`
  __device__ static uint32_t sf_col(uint32_t it, int s) {
    return (uint32_t)NB + (kSfPerStage ? (uint32_t)s : it % (uint32_t)kSfBufs) * kSfCols;
  }
};

// Epilogue of one warp (q = lane quadrant, h = column half) when the next
// layer has a low-rank branch. Per tile:
//   1. drain the accumulator (bf16-packed) and release it to the MMA issuer;
//   2. write the next layer's codes and scales (epilogue_encode_next);
//   3. stage the band's two 64-column boxes b (rows of this CTA, bf16 Y) in
//      the warp's own boxes -- the four warps of a half form one 128 x 64
//      K-major operand per b -- store them to Y if asked, and report each to
//      the even CTA (ych_full[h][b]). One thread (even CTA, warp q = 0, h = 1)
//      issues the T' MMAs of every chunk in the order (b, h) = (0,0), (0,1),
//      (1,0), (1,1): D (TMEM columns kTpCol.., both CTAs) += Y chunk x L1p'
//      chunk^T, committing each chunk to ych_empty[h][b] and the tile to
//      tp_full;
//   4. the warps of half 0 read T' (their 32 lanes) and write the tile's fp32
//      partial to nq.tp_ws[tile column][row][:], then report tp_empty.
// Warps q = 0 of each CTA TMA-load the L1p' columns of their half (the B rows
// of this CTA: next_rank/2 of them) for each tile into l1_full[h], after the
// previous tile's T' MMAs have completed. Each barrier completes once per
// tile, so parity waits cannot alias across tiles.
template <class C>
__device__ __forceinline__ void epilogue_next_lowrank(
    unsigned char* smem, uint32_t tmem, uint32_t crank, bool leader, int q, int h, int lane, int cluster,
    int nclusters, int ntiles, int tiles_n, int M, int N, const NextQuant& nq, const float2* rcp_tbl,
    const void* tm_y, const void* tm_l1n, bool store_y, uint64_t* acc_full, uint64_t* acc_empty,
    uint64_t* ych_full, uint64_t* ych_empty, uint64_t* tp_full, uint64_t* tp_empty, uint64_t* l1_full,
    uint64_t* tp_drain) {
  const int rh = nq.next_rank / 2;                              // L1p' rows per CTA (B rows of the pair MMA)
  const uint32_t l1_bytes = 2u * (uint32_t)rh * 128u;
  unsigned char* l1buf = smem + C::kL1Offset + h * C::kL1Half;
  const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
  const uint32_t tp_empty_leader = mapa_shared(smem_u32(tp_empty), 0);
  const bool loader = q == 0 && lane == 0;
  const bool issuer = leader && q == 0 && h == 1 && lane == 0;
  const uint32_t idesc_tp = idesc_bf16(kPairBM, nq.next_rank);
  uint32_t l1_issued = 0;
  auto load_l1 = [&](int tile) {
    const int n0 = (tile % tiles_n) * 256 + h * 128;
    ++l1_issued;
    mbar_arrive_expect_tx(l1_full + h, l1_bytes);
    tma_load_2d(l1buf, tm_l1n, l1_full + h, n0, (int)crank * rh);
    tma_load_2d(l1buf + rh * 128, tm_l1n, l1_full + h, n0 + 64, (int)crank * rh);
  };
  if (loader && cluster < ntiles) load_l1(cluster);
  bool ok = true;
  uint32_t tcount = 0;
  for (int tile = cluster; tile < ntiles && ok; tile += nclusters, ++tcount) {
    const int m0 = (tile / tiles_n) * kPairBM + 128 * (int)crank;
    const int n0 = (tile % tiles_n) * 256;
    const uint32_t par = tcount & 1u;
    const float4 inv4 = epilogue_inv_factors(nq, n0 + h * 128, lane);
    ok = mbar_wait(acc_full, par, kDevErrTimeoutAccum) && !device_error_set();
    ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;   // one decision per warp
    tc_fence_after();
    if (!ok) break;
    const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * 128);
    uint32_t p[64];
    epilogue_drain_pack<4>(taddr, p);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_remote(acc_empty_leader);
    epilogue_encode_next<2>(p, nq, rcp_tbl, inv4, m0 + 32 * q, n0 + h * 128, M, N, lane);
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      unsigned char* box = smem + C::kEpiOffset + ((h * 2 + b) * 4 + q) * kEpiBoxBytes;
      if (lane == 0) {
        // the box's previous T' MMAs and its previous Y store have read it
        if (tcount > 0 && !mbar_wait(ych_empty + h * 2 + b, par ^ 1u, kDevErrTimeoutNext)) ok = false;
        bulk_wait_read<1>();
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      epilogue_stage_box(&p[32 * b], box, lane);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (q == 0 && b == 0 && !mbar_wait(l1_full + h, par, kDevErrTimeoutNext)) ok = false;
        if (ok) mbar_arrive_remote(mapa_shared(smem_u32(ych_full + h * 2 + b), 0));
        if (store_y && m0 + 32 * q < M) {
          tma_store_2d_evict_first(tm_y, box, n0 + h * 128 + 64 * b, m0 + 32 * q);
        }
        bulk_commit();   // one group per box, stored or not, so that bulk_wait_read<1> keeps its meaning
      }
      if (issuer && ok) {
#pragma unroll 1
        for (int hh = 0; hh < 2 && ok; ++hh) {
          if (!mbar_wait(ych_full + hh * 2 + b, par, kDevErrTimeoutNext)) {
            ok = false;
            break;
          }
          if (b == 0 && hh == 0 && tcount > 0 && !mbar_wait(tp_empty, par ^ 1u, kDevErrTimeoutNext)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = smem_desc(smem_u32(smem + C::kEpiOffset + (hh * 2 + b) * 4 * kEpiBoxBytes), 16, 1024,
                                        kSwizzle128B);
          const uint64_t bd = smem_desc(smem_u32(smem + C::kL1Offset + hh * C::kL1Half + b * rh * 128), 16, 1024,
                                        kSwizzle128B);
#pragma unroll
          for (int j = 0; j < 4; ++j)   // 16 bf16 (32 bytes) of the chunk's 64 columns per MMA
            mma_bf16_pair(tmem + C::kTpCol, ad + 2u * j, bd + 2u * j, idesc_tp, (b | hh | j) != 0 ? 1u : 0u);
          tc_commit_pair(ych_empty + hh * 2 + b, 0x3);
        }
        if (ok && b == 1) tc_commit_pair(tp_full, 0x3);
      }
      __syncwarp();
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
    }
    if (!ok) break;
    // the tile's T' partial
    if (h == 0) {
      ok = mbar_wait(tp_full, par, kDevErrTimeoutNext);
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      tc_fence_after();
      if (!ok) break;
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) + C::kTpCol, v);
      tmem_ld_wait();
      const int row = m0 + 32 * q + lane;
      if (row < M) {
        float4* dst = reinterpret_cast<float4*>(nq.tp_ws + ((size_t)(tile % tiles_n) * (size_t)M + (size_t)row) *
                                                               (size_t)nq.next_rank);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (4 * i < nq.next_rank)
            dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                 __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(tp_empty_leader);
    }
    // the next tile's L1p' columns, once this tile's T' MMAs are done with the buffer
    if (q == 0) {
      bool lok = true;
      if (lane == 0 && tile + nclusters < ntiles) {
        if (h == 1) lok = mbar_wait(tp_full, par, kDevErrTimeoutNext);
        if (lok) load_l1(tile + nclusters);
      }
      ok = __shfl_sync(0xFFFFFFFFu, lok ? 1 : 0, 0) != 0;
    }
  }
  // leave no TMA load of L1p' in flight (the last one was consumed already
  // unless the loop stopped early; waiting on a completed phase returns at once)
  if (loader && l1_issued > 0) mbar_drain(l1_full + h, (l1_issued - 1u) & 1u);
  // and no T' MMA running when TMEM is freed
  if (issuer && tcount + (ok ? 0u : 1u) > 0) {
    tc_commit_pair(tp_drain, 0x1);
    mbar_drain(tp_drain, 0);
  }
}

// Launched with a cluster dimension of (2, 1, 1).
// tm_qr / tm_l2 boxes are 128 rows (NB = 256) or 64 rows (NB = 384).
// tm_sfa / tm_sfb view a native scale buffer as 3-D uint8
// [row blocks][K/64 * 2 chunks][256 bytes]; box {256, 8, 1 | NB/128} (4 atoms per row block).
// QNEXT: the epilogue also quantizes Y for the next layer (svdq_gemm_qnext.cuh),
// and stores Y itself only when store_y is set.
// QLR (with QNEXT): the next layer has a low-rank branch; tm_l1n views its
// L1p' [next_rank][N] bf16 with boxes of 64 columns x next_rank/2 rows.
template <int NB, bool QNEXT = false, bool QLR = false>
__global__ void __launch_bounds__(kGemmThreads, 1) svdq_gemm_pair_kernel(
    const __grid_constant__ CUtensorMap tm_qx, const __grid_constant__ CUtensorMap tm_qr,
    const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
    const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_l2,
    const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_l1n, int M, int N, int K,
    int rank, NextQuant nq, int store_y) {
  static_assert(!QNEXT || NB == 256, "the next layer's quantization runs on 256 x 256 tiles");
  static_assert(!QLR || QNEXT, "the next layer's down-projection comes with its quantization");
  using C = PairCfg<NB, QLR>;
  constexpr int STAGES = C::kStages;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* empty = full + STAGES;
  uint64_t* sf_ready = empty + STAGES;      // even CTA: both CTAs' scale warps report here
  uint64_t* acc_full = sf_ready + STAGES;
  uint64_t* acc_empty = acc_full + 1;       // even CTA: both CTAs' epilogue warps report here
  uint64_t* mma_drain = acc_empty + 1;
  // QLR only: chunk (h, b) of the staged Y is in both CTAs (even CTA, 8 warp
  // arrivals) / has been read by its T' MMAs (both CTAs, commit); the tile's
  // T' partial is complete (both CTAs, commit) / has been read out (even CTA,
  // 8 warp arrivals); this CTA's L1p' half h has landed
  uint64_t* ych_full = mma_drain + 1;       // [h * 2 + b]
  uint64_t* ych_empty = ych_full + 4;       // [h * 2 + b]
  uint64_t* tp_full = ych_empty + 4;
  uint64_t* tp_empty = tp_full + 1;
  uint64_t* l1_full = tp_empty + 1;         // [h]
  uint64_t* tp_drain = l1_full + 2;         // the T' issuer's MMAs have all completed (before TMEM is freed)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tp_drain + 1);

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
    if (QLR) {
      for (int i = 0; i < 4; ++i) {
        mbar_init(ych_full + i, 2 * 4);
        mbar_init(ych_empty + i, 1);
      }
      mbar_init(tp_full, 1);
      mbar_init(tp_empty, 2 * 4);
      mbar_init(l1_full, 1);
      mbar_init(l1_full + 1, 1);
      mbar_init(tp_drain, 1);
    }
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
    if (QLR) prefetch_tmap(&tm_l1n);
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
      if (device_error_set()) {   // let the copies this thread issued land before the CTA exits
        for (uint32_t j = it > (uint32_t)STAGES ? it - STAGES : 0u; j < it; ++j)
          mbar_drain(full + j % STAGES, (j / STAGES) & 1u);
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
        mbar_drain(mma_drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3, h = warp >> 2;
    unsigned char* box = smem + C::kEpiOffset + warp * kEpiBoxBytes;
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
    if (lane == 0 && (!QNEXT || store_y)) prefetch_tmap(&tm_y);
    if constexpr (QLR) {
      epilogue_next_lowrank<C>(smem, tmem, crank, leader, q, h, lane, cluster, nclusters, ntiles, tiles_n, M, N, nq,
                               rcp_tbl, &tm_y, &tm_l1n, store_y != 0, acc_full, acc_empty, ych_full, ych_empty,
                               tp_full, tp_empty, l1_full, tp_drain);
    } else {
    uint32_t tcount = 0;
    for (int tile = cluster; tile < ntiles; tile += nclusters, ++tcount) {
      const int m0 = (tile / tiles_n) * kPairBM + 128 * (int)crank;
      const int n0 = (tile % tiles_n) * NB;
      const float4 inv4 = QNEXT ? epilogue_inv_factors(nq, n0 + h * 128, lane) : make_float4(0.f, 0.f, 0.f, 0.f);
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
          epilogue_quantize_next<2>(p, box, nq, rcp_tbl, inv4, &tm_y, store_y != 0, m0 + 32 * q, n0 + h * 128, M, N,
                                    lane);
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
