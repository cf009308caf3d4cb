// The W4A4 GEMM of the SVDQuant layer on 5th-generation tensor cores:
//   Y = bf16( deq(Qx) deq(Qr)^T  +  T L2t^T )
// (devpress.csdn.net SVDQuant walkthrough, eq. (2) and eq. (5); Fig. 6: the
// up-projection shares the 4-bit GEMM's output). The FP4 products run as
// tcgen05 block-scaled MMAs (kind::mxf4nvf4, one UE4M3 scale per 16 K-elements)
// into an fp32 TMEM accumulator; the rank-r up-projection then runs as bf16
// MMAs (kind::f16) into the same accumulator, so the 16-bit branch adds no pass
// over Y.
//
// This single-CTA kernel serves every N that is a multiple of 128; the CTA-pair
// kernel (svdq_gemm_pair.cuh) takes over when N is a multiple of 256.
//
// Persistent kernel: one CTA per SM walks output tiles of BM x BN = 128 x 256
// (tile = blockIdx.x, blockIdx.x + gridDim.x, ...). Every tile is a sequence
// of k-tiles ("items"): K/256 FP4 items, then ceil(r/64) low-rank items, all
// through one ring of STAGES shared-memory stages. Warp roles (448 threads):
//   warps 0-7   epilogue: warp w drains accumulator lanes 32(w%4).. and columns
//               128(w/4).., releases the accumulator, then writes Y through
//               128B-swizzled boxes and TMA stores while the next tile runs
//   warp 8      producer: TMA loads of the Qx / Qr (then T / L2t) k-tile rows
//               and bulk copies of the Sx / Sr scale atoms into the ring
//   warp 9      TMEM allocation; one lane issues the MMAs of each item once its
//               scales are in TMEM, and releases each ring stage (with its
//               TMEM scale buffer) and the accumulator with tcgen05.commit
//   warps 10-13 scale warps: copy each item's scale atoms into the TMEM scale
//               buffer of its ring stage with tcgen05.st (svdq_gemm_common.cuh)
// Every wait is bounded (svdq::mbar_wait); on a timeout the kernel records a
// device error word and every role drains and returns.
#pragma once

#include <cuda_bf16.h>

#include "svdq_gemm_common.cuh"
#include "svdq_ptx.cuh"

namespace svdq {

constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;
constexpr int kStageA = kGemmBM * kGemmBKBytes;   // 16 KB (also T: 128 x 64 bf16)
constexpr int kStageB = kGemmBN * kGemmBKBytes;   // 32 KB (also L2t: 256 x 64 bf16)
constexpr int kStageSfa = kGemmKBPerStage * kSfAtomBytes;
constexpr int kStageSfb = 2 * kGemmKBPerStage * kSfAtomBytes;
constexpr int kStageBytes = kStageA + kStageB + kStageSfa + kStageSfb;   // 54 KB

template <int STAGES>
struct GemmSmem {
  static constexpr int kEpiOffset = STAGES * kStageBytes;
  static constexpr int kBarOffset = kEpiOffset + kGemmEpiWarps * kEpiBoxBytes;
  static constexpr int kBytes = kBarOffset + 512 + 1024;   // barriers + alignment slack
};

template <int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1) svdq_gemm_kernel(
    const __grid_constant__ CUtensorMap tm_qx, const __grid_constant__ CUtensorMap tm_qr,
    const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_l2,
    const __grid_constant__ CUtensorMap tm_y, const uint8_t* __restrict__ Sx, const uint8_t* __restrict__ Sr,
    int M, int N, int K, int rank) {
  using L = GemmSmem<STAGES>;
  static_assert(STAGES <= kMaxSfBufs, "one TMEM scale buffer per ring stage");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOffset);
  uint64_t* empty = full + STAGES;
  uint64_t* sf_ready = empty + STAGES;
  uint64_t* acc_full = sf_ready + STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* mma_drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = (N + kGemmBN - 1) / kGemmBN;
  const int ntiles = ((M + kGemmBM - 1) / kGemmBM) * tiles_n;
  const int kb_total = K >> 6;
  const int n_fp4_kt = (kb_total + kGemmKBPerStage - 1) / kGemmKBPerStage;
  const int n_lr_kt = (rank + kGemmLrK - 1) / kGemmLrK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < STAGES; ++b) mbar_init(sf_ready + b, kSfWarps);
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kGemmEpiWarps);
    mbar_init(mma_drain, 1);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&tm_qx);
    prefetch_tmap(&tm_qr);
    if (rank > 0) {
      prefetch_tmap(&tm_t);
      prefetch_tmap(&tm_l2);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dependency_wait();     // the previous kernel's outputs (Qx, Sx, T) are complete
  grid_launch_dependents();

  if (warp == kProducerWarp) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int m0 = (tile / tiles_n) * kGemmBM, n0 = (tile % tiles_n) * kGemmBN;
        const bool half = n0 + kGemmBN > N;    // only the first 128 B rows exist
        const uint8_t* sfa_src = Sx + (size_t)(m0 >> 7) * kb_total * kSfAtomBytes;
        const uint8_t* sfb_src = Sr + (size_t)(n0 >> 7) * kb_total * kSfAtomBytes;
        for (int kt = 0; kt < n_fp4_kt + n_lr_kt; ++kt, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(empty + s, ((it / STAGES) & 1u) ^ 1u, kDevErrTimeoutEmpty)) {
            ok = false;
            break;
          }
          unsigned char* sa = smem + s * kStageBytes;
          unsigned char* sb = sa + kStageA;
          if (kt < n_fp4_kt) {
            unsigned char* sfa = sb + kStageB;
            unsigned char* sfb = sfa + kStageSfa;
            const int kbs = min(kGemmKBPerStage, kb_total - kt * kGemmKBPerStage);
            const uint32_t sf_bytes = (uint32_t)kbs * kSfAtomBytes;
            mbar_arrive_expect_tx(full + s, (uint32_t)(kStageA + kStageB) + sf_bytes * (half ? 2u : 3u));
            tma_load_2d(sa, &tm_qx, full + s, kt * kGemmBKBytes, m0);
            tma_load_2d(sb, &tm_qr, full + s, kt * kGemmBKBytes, n0);
            const size_t off = (size_t)kt * kGemmKBPerStage * kSfAtomBytes;
            bulk_load(sfa, sfa_src + off, sf_bytes, full + s);
            bulk_load(sfb, sfb_src + off, sf_bytes, full + s);
            if (!half)
              bulk_load(sfb + kStageSfb / 2, sfb_src + (size_t)kb_total * kSfAtomBytes + off, sf_bytes, full + s);
          } else {
            const int c = kt - n_fp4_kt;
            mbar_arrive_expect_tx(full + s, (uint32_t)(kStageA + kStageB));
            tma_load_2d(sa, &tm_t, full + s, c * kGemmLrK, m0);
            tma_load_2d(sb, &tm_l2, full + s, c * kGemmLrK, n0);
          }
        }
      }
      if (device_error_set()) {
        // Another role gave up: let the copies this thread issued land before
        // the CTA exits (bounded; only the last STAGES stages can be in flight).
        for (uint32_t j = it > (uint32_t)STAGES ? it - STAGES : 0u; j < it; ++j)
          mbar_drain(full + j % STAGES, (j / STAGES) & 1u);
      }
    }
  } else if (warp >= kSfWarp0) {
    // ------------------------------------------------------------------ scale warps
    const int q = warp & 3;
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
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
          const unsigned char* sfa = smem + s * kStageBytes + kStageA + kStageB;
          const unsigned char* sfb = sfa + kStageSfa;
          scales_to_tmem(tmem, q, lane, sfa, sfb, sfb + kStageSfb / 2, sf_buf_col(s));
          tmem_st_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sf_ready + s);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++tcount) {
        const int n0 = (tile % tiles_n) * kGemmBN;
        const bool half = n0 + kGemmBN > N;
        const uint32_t idesc = idesc_nvfp4(kGemmBM, half ? kGemmBN / 2 : kGemmBN);
        const uint32_t idesc_lr = idesc_bf16(kGemmBM, half ? kGemmBN / 2 : kGemmBN);
        if (!mbar_wait(acc_empty, (tcount & 1u) ^ 1u, kDevErrTimeoutAccum)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kt = 0; kt < n_fp4_kt + n_lr_kt; ++kt, ++it) {
          const int s = it % STAGES;
          // the scale warps saw stage s full and put its scales in TMEM
          if (!mbar_wait(sf_ready + s, (it / STAGES) & 1u, kDevErrTimeoutScales)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * kStageBytes);
          const uint32_t sb = sa + kStageA;
          if (kt < n_fp4_kt) {
            const uint32_t sfa = tmem + sf_buf_col(s);
            const uint32_t sfb = sfa + 4 * kGemmKBPerStage;
            const int kbs = min(kGemmKBPerStage, kb_total - kt * kGemmKBPerStage);
            for (int kb = 0; kb < kbs; ++kb) {
              const uint64_t ad = smem_desc(sa + kb * 32, 16, 1024, kSwizzle128B);
              const uint64_t bd = smem_desc(sb + kb * 32, 16, 1024, kSwizzle128B);
              mma_nvfp4(tmem, ad, bd, idesc, sfa + 4 * kb, sfb + 8 * kb, (kt | kb) != 0 ? 1u : 0u);
            }
          } else {
            const int c = kt - n_fp4_kt;
            const int k16 = min(kGemmLrK, rank - c * kGemmLrK) / 16;
            for (int j = 0; j < k16; ++j) {
              const uint64_t ad = smem_desc(sa + j * 32, 16, 1024, kSwizzle128B);
              const uint64_t bd = smem_desc(sb + j * 32, 16, 1024, kSwizzle128B);
              mma_bf16(tmem, ad, bd, idesc_lr, 1u);
            }
          }
          tc_commit(empty + s);     // ring stage s and its scale buffer are free once these MMAs ran
        }
        tc_commit(acc_full);        // the tile's accumulator is complete
      }
      if (!ok) {
        // Gave up: wait (bounded) for the MMAs already issued before TMEM is freed.
        tc_commit(mma_drain);
        mbar_drain(mma_drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3, h = warp >> 2;
    unsigned char* box = smem + L::kEpiOffset + warp * kEpiBoxBytes;
    if (lane == 0) prefetch_tmap(&tm_y);
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tcount) {
      const int m0 = (tile / tiles_n) * kGemmBM, n0 = (tile % tiles_n) * kGemmBN;
      const bool ok = mbar_wait(acc_full, tcount & 1u, kDevErrTimeoutAccum);
      tc_fence_after();
      if (!ok || device_error_set()) break;
      uint32_t p[64];
      epilogue_drain_pack<4>(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * 128), p);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);   // accumulator drained: the next tile may start
      const int col0 = n0 + h * 128;
      if (col0 >= N) continue;                 // second half of a 128-wide last column tile
      epilogue_store_band<2>(p, box, &tm_y, col0, m0 + 32 * q, lane, true);
    }
    if (lane == 0) bulk_wait<0>();   // every store of this warp has completed
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace svdq
