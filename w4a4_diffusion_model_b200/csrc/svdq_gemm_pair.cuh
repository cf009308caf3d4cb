// The W4A4 GEMM on CTA pairs: one tcgen05 MMA (cta_group::2) spans the two
// SMs of a cluster of 2, computing a 256 x 256 tile of
//   Y = bf16( deq(Qx) deq(Qr)^T  +  T L2t^T )
// (devpress.csdn.net SVDQuant walkthrough, eq. (2), eq. (5) and Fig. 6).
// Each CTA of the pair stages its own 128 rows of the A operand (Qx, then T)
// and its own 128 rows of the B operand (Qr, then L2t), so a pair reads 2/3 of
// the operand bytes two independent 128 x 256 tiles would. Each CTA stages
// the A scales of its 128 rows and the B scales of all 256 columns; the even
// CTA's tcgen05.cp (cta_group::2) copies each CTA's scales into its own TMEM.
//
// Persistent: cluster c walks pair tiles c, c + clusters, ... Roles per CTA
// (320 threads), identical in both CTAs except where noted:
//   warps 0-7  epilogue: drain this CTA's 128 x 256 fp32 accumulator from TMEM,
//              release it to the even CTA's MMA issuer, then convert to bf16
//              and write Y through 128B-swizzled TMA-store boxes
//   warp 8     producer: TMA loads (cta_group::2 form, completion counted on
//              the even CTA's barrier) of this CTA's A / B k-tile rows and of
//              the scale atoms; the even CTA also arms the expected byte count
//              of both CTAs
//   warp 9     TMEM allocation (both CTAs); in the even CTA one lane issues the
//              scale copies and MMAs, releasing stages of both CTAs with one
//              multicast tcgen05.commit
// Every wait is bounded; on a timeout the kernel records a device error word,
// every role stops, and both CTAs still meet at the final cluster barrier.
#pragma once

#include <cuda_bf16.h>

#include "svdq_gemm.cuh"
#include "svdq_ptx.cuh"

namespace svdq {

constexpr int kPairBM = 256;                          // M rows per pair tile (128 per CTA)
constexpr int kPairBN = 256;                          // N columns per pair tile (B rows: 128 per CTA)
constexpr int kPairStageA = 128 * kGemmBKBytes;       // 16 KB: this CTA's 128 Qx rows (or T rows)
constexpr int kPairStageB = 128 * kGemmBKBytes;       // 16 KB: this CTA's 128 Qr rows (or L2t rows)
constexpr int kPairStageSfa = kGemmKBPerStage * kSfAtomBytes;       // 2 KB
constexpr int kPairStageSfb = 2 * kGemmKBPerStage * kSfAtomBytes;   // 4 KB (both 128-row halves of N)
constexpr int kPairStageBytes = kPairStageA + kPairStageB + kPairStageSfa + kPairStageSfb;   // 38 KB
constexpr uint32_t kPairSfCols = 4 * kGemmKBPerStage * 3;   // A scales + B scales of one k-tile
constexpr uint32_t kPairSfaCol = kGemmBN;                    // after the 256 accumulator columns
constexpr uint32_t kPairSfbCol = kGemmBN + 4 * kGemmKBPerStage;

template <int STAGES>
struct PairSmem {
  static constexpr int kEpiOffset = STAGES * kPairStageBytes;
  static constexpr int kBarOffset = kEpiOffset + kGemmEpiWarps * kEpiBoxBytes;
  static constexpr int kBytes = kBarOffset + 256 + 1024;
};

// Launched with a cluster dimension of (2, 1, 1).
// tm_sfa / tm_sfb view a native scale buffer as 4-D uint8
// [row blocks][K/64 atoms][32 lines][16 bytes]; box {16, 32, 4, 1|2}.
template <int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1) svdq_gemm_pair_kernel(
    const __grid_constant__ CUtensorMap tm_qx, const __grid_constant__ CUtensorMap tm_qr,
    const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
    const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_l2,
    const __grid_constant__ CUtensorMap tm_y, int M, int N, int K, int rank) {
  using L = PairSmem<STAGES>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOffset);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 1;
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
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * kGemmEpiWarps);   // both CTAs' epilogue warps (used in the even CTA)
    mbar_init(mma_drain, 1);
    fence_mbar_init();
  }
  if (warp == kGemmEpiWarps + 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == kGemmEpiWarps && lane == 0) {
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

  if (warp == kGemmEpiWarps) {
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
          const uint32_t bar = mapa_shared(smem_u32(full + s), 0);   // counted on the even CTA
          if (kt < n_fp4_kt) {
            unsigned char* sfa = sb + kPairStageB;
            unsigned char* sfb = sfa + kPairStageSfa;
            if (leader) mbar_arrive_expect_tx(full + s, 2u * (uint32_t)kPairStageBytes);
            tma_load_2d_pair(sa, &tm_qx, bar, kt * kGemmBKBytes, m0);
            tma_load_2d_pair(sb, &tm_qr, bar, kt * kGemmBKBytes, n0 + 128 * (int)crank);
            tma_load_4d_pair(sfa, &tm_sfa, bar, 0, 0, kt * kGemmKBPerStage, m0 >> 7);
            tma_load_4d_pair(sfb, &tm_sfb, bar, 0, 0, kt * kGemmKBPerStage, n0 >> 7);
          } else {
            const int c = kt - n_fp4_kt;
            if (leader) mbar_arrive_expect_tx(full + s, 2u * (uint32_t)(kPairStageA + kPairStageB));
            tma_load_2d_pair(sa, &tm_t, bar, c * kGemmLrK, m0);
            tma_load_2d_pair(sb, &tm_l2, bar, c * kGemmLrK, n0 + 128 * (int)crank);
          }
        }
      }
      if (device_error_set() && leader) {
        // Another role gave up: let the copies counted here land before exit.
        for (uint32_t j = it > (uint32_t)STAGES ? it - STAGES : 0u; j < it; ++j)
          mbar_wait(full + j % STAGES, (j / STAGES) & 1u, kDevErrTimeoutFull);
      }
    }
  } else if (warp == kGemmEpiWarps + 1) {
    if (lane == 0 && leader) {
      // ---------------------------------------------------------------- MMA issuer (even CTA)
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      const uint32_t idesc = idesc_nvfp4(kPairBM, kPairBN);
      const uint32_t idesc_lr = idesc_bf16(kPairBM, kPairBN);
      for (int tile = cluster; tile < ntiles && ok; tile += nclusters, ++tcount) {
        if (!mbar_wait(acc_empty, (tcount & 1u) ^ 1u, kDevErrTimeoutAccum)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kt = 0; kt < n_fp4_kt + n_lr_kt; ++kt, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(full + s, (it / STAGES) & 1u, kDevErrTimeoutFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * kPairStageBytes);
          const uint32_t sb = sa + kPairStageA;
          if (kt < n_fp4_kt) {
            const uint32_t sfa = sb + kPairStageB;
            const uint32_t sfb = sfa + kPairStageSfa;
            const uint32_t col = (it & 1u) * kPairSfCols;   // alternate scale buffers
            const int kbs = min(kGemmKBPerStage, kb_total - kt * kGemmKBPerStage);
            for (int kb = 0; kb < kbs; ++kb) {
              tmem_cp_pair_32x128b_x4(tmem + kPairSfaCol + col + 4 * kb,
                                      smem_desc(sfa + kb * kSfAtomBytes, 16, 128, kSwizzleNone));
              tmem_cp_pair_32x128b_x4(tmem + kPairSfbCol + col + 8 * kb,
                                      smem_desc(sfb + kb * kSfAtomBytes, 16, 128, kSwizzleNone));
              tmem_cp_pair_32x128b_x4(tmem + kPairSfbCol + col + 8 * kb + 4,
                                      smem_desc(sfb + kPairStageSfb / 2 + kb * kSfAtomBytes, 16, 128, kSwizzleNone));
            }
            for (int kb = 0; kb < kbs; ++kb) {
              const uint64_t ad = smem_desc(sa + kb * 32, 16, 1024, kSwizzle128B);
              const uint64_t bd = smem_desc(sb + kb * 32, 16, 1024, kSwizzle128B);
              mma_nvfp4_pair(tmem, ad, bd, idesc, tmem + kPairSfaCol + col + 4 * kb,
                             tmem + kPairSfbCol + col + 8 * kb, (kt | kb) != 0 ? 1u : 0u);
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
          tc_commit_pair(empty + s, 0x3);   // stage s of both CTAs is free once these MMAs read it
        }
        tc_commit_pair(acc_full, 0x3);      // both halves of the tile's accumulator are complete
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
    const uint32_t box_addr = smem_u32(box);
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
    if (lane == 0) prefetch_tmap(&tm_y);
    uint32_t tcount = 0;
    for (int tile = cluster; tile < ntiles; tile += nclusters, ++tcount) {
      const int m0 = (tile / tiles_n) * kPairBM + 128 * (int)crank;
      const int n0 = (tile % tiles_n) * kPairBN;
      const bool ok = mbar_wait(acc_full, tcount & 1u, kDevErrTimeoutAccum);
      tc_fence_after();
      if (!ok || device_error_set()) break;
      uint32_t v[128];
      const uint32_t base = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * 128);
      tmem_ld_32x32b_x32(base + 0, *reinterpret_cast<uint32_t(*)[32]>(v + 0));
      tmem_ld_32x32b_x32(base + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
      tmem_ld_32x32b_x32(base + 64, *reinterpret_cast<uint32_t(*)[32]>(v + 64));
      tmem_ld_32x32b_x32(base + 96, *reinterpret_cast<uint32_t(*)[32]>(v + 96));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(acc_empty_leader);   // this warp's part of the accumulator is drained
      const int col0 = n0 + h * 128;
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t p[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int e = 64 * b + 8 * c + 2 * i;
            const __nv_bfloat162 bb = __floats2bfloat162_rn(__uint_as_float(v[e]), __uint_as_float(v[e + 1]));
            p[i] = *reinterpret_cast<const uint32_t*>(&bb);
          }
          const uint32_t addr = box_addr + lane * 128 + ((c ^ (lane & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(p[0]), "r"(p[1]), "r"(p[2]),
                       "r"(p[3])
                       : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && m0 + 32 * q < M) {
          tma_store_2d(&tm_y, box, col0 + 64 * b, m0 + 32 * q);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait<0>();
  }

  tc_fence_before();
  cluster_sync();   // no CTA leaves while its peer may still signal its barriers
  if (warp == kGemmEpiWarps + 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace svdq
