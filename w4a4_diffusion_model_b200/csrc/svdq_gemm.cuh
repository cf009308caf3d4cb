// The W4A4 GEMM of the SVDQuant layer on 5th-generation tensor cores:
//   Y = bf16( deq(Qx) deq(Qr)^T  +  T L2t^T )
// (devpress.csdn.net SVDQuant walkthrough, eq. (2) and eq. (5); Fig. 6: the
// up-projection shares the 4-bit GEMM's output). The FP4 products run as
// tcgen05 block-scaled MMAs (kind::mxf4nvf4, one UE4M3 scale per 16 K-elements)
// into an fp32 TMEM accumulator; the rank-r up-projection then runs as bf16
// MMAs (kind::f16) into the same accumulator, so the 16-bit branch adds no pass
// over Y.
//
// One CTA computes one BM x BN = 128 x 128 tile of Y with warp-specialized
// roles (192 threads):
//   warps 0-3  epilogue: TMEM -> registers -> bf16 -> global (warp w owns
//              accumulator lanes 32w..32w+31, i.e. rows m0+32w..)
//   warp 4     producer: TMA loads of the Qx/Qr tiles (128 B K-rows, 128B
//              swizzle) and bulk copies of the Sx/Sr scale atoms into a ring
//              of STAGES shared-memory stages; TMA loads of the T / L2t tiles
//   warp 5     TMEM allocation; one lane issues tcgen05.cp (scales -> TMEM)
//              and the MMAs, and commits stage releases / accumulator-ready.
// Every wait is bounded (svdq::mbar_wait); on a timeout the kernel records a
// device error word and every role drains and returns.
#pragma once

#include <cuda_bf16.h>

#include "svdq_ptx.cuh"

namespace svdq {

constexpr int kGemmBM = 128;
constexpr int kGemmBN = 128;
constexpr int kGemmBKBytes = 128;                 // 256 FP4 elements per stage row
constexpr int kGemmKBPerStage = 4;                // 64-element MMA K blocks per stage
constexpr int kGemmThreads = 192;

constexpr int kTileABytes = kGemmBM * kGemmBKBytes;   // 16 KB
constexpr int kTileBBytes = kGemmBN * kGemmBKBytes;   // 16 KB
constexpr int kSfAtomBytes = 512;                     // 128 rows x 4 scales

// TMEM columns: accumulator [0, BN), scale factors of A then B after it.
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kTmemSfaCol = kGemmBN;
constexpr uint32_t kTmemSfbCol = kGemmBN + 4 * kGemmKBPerStage;

template <int STAGES, int RANK>
struct GemmSmem {
  static constexpr int kStageBytes = kTileABytes + kTileBBytes + 2 * kGemmKBPerStage * kSfAtomBytes;
  static constexpr int kLrSlabA = kGemmBM * 32;   // one 16-wide bf16 K slab of T: 128 rows x 32 B
  static constexpr int kLrSlabB = kGemmBN * 32;
  static constexpr int kLrBytes = (RANK / 16) * (kLrSlabA + kLrSlabB);
  static constexpr int kBarOffset = STAGES * kStageBytes + kLrBytes;
  static constexpr int kBytes = kBarOffset + 256 + 1024;   // barriers + alignment slack
};

template <int STAGES, int RANK>
__global__ void __launch_bounds__(kGemmThreads, 1) svdq_gemm_kernel(
    const __grid_constant__ CUtensorMap tm_qx, const __grid_constant__ CUtensorMap tm_qr,
    const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_l2,
    const uint8_t* __restrict__ Sx, const uint8_t* __restrict__ Sr, __nv_bfloat16* __restrict__ Y, int M, int N,
    int K) {
  using L = GemmSmem<STAGES, RANK>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOffset);
  uint64_t* empty = full + STAGES;
  uint64_t* lr_full = empty + STAGES;
  uint64_t* acc_full = lr_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  unsigned char* lr_a = smem + STAGES * L::kStageBytes;
  unsigned char* lr_b = lr_a + (RANK / 16) * L::kLrSlabA;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kGemmBN, m0 = blockIdx.y * kGemmBM;
  const int kb_total = K >> 6;
  const int num_kt = (kb_total + kGemmKBPerStage - 1) / kGemmKBPerStage;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    mbar_init(lr_full, 1);
    mbar_init(acc_full, 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&tm_qx);
    prefetch_tmap(&tm_qr);
    if (RANK > 0) {
      prefetch_tmap(&tm_t);
      prefetch_tmap(&tm_l2);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      if (RANK > 0) {
        mbar_arrive_expect_tx(lr_full, (uint32_t)L::kLrBytes);
        for (int j = 0; j < RANK / 16; ++j) {
          tma_load_2d(lr_a + j * L::kLrSlabA, &tm_t, lr_full, j * 16, m0);
          tma_load_2d(lr_b + j * L::kLrSlabB, &tm_l2, lr_full, j * 16, n0);
        }
      }
      const uint8_t* sfa_src = Sx + (size_t)(m0 >> 7) * kb_total * kSfAtomBytes;
      const uint8_t* sfb_src = Sr + (size_t)(n0 >> 7) * kb_total * kSfAtomBytes;
      for (int kt = 0; kt < num_kt; ++kt) {
        const int s = kt % STAGES;
        const uint32_t ph = (uint32_t)(kt / STAGES) & 1u;
        if (!mbar_wait(empty + s, ph ^ 1u, kDevErrTimeoutEmpty)) break;
        const int kbs = min(kGemmKBPerStage, kb_total - kt * kGemmKBPerStage);
        unsigned char* st = smem + s * L::kStageBytes;
        unsigned char* sa = st;
        unsigned char* sb = st + kTileABytes;
        unsigned char* sfa = sb + kTileBBytes;
        unsigned char* sfb = sfa + kGemmKBPerStage * kSfAtomBytes;
        mbar_arrive_expect_tx(full + s, (uint32_t)(kTileABytes + kTileBBytes + 2 * kbs * kSfAtomBytes));
        tma_load_2d(sa, &tm_qx, full + s, kt * kGemmBKBytes, m0);
        tma_load_2d(sb, &tm_qr, full + s, kt * kGemmBKBytes, n0);
        bulk_load(sfa, sfa_src + (size_t)kt * kGemmKBPerStage * kSfAtomBytes, kbs * kSfAtomBytes, full + s);
        bulk_load(sfb, sfb_src + (size_t)kt * kGemmKBPerStage * kSfAtomBytes, kbs * kSfAtomBytes, full + s);
      }
      if (device_error_set()) {
        // Another role gave up: let the copies this thread issued land before
        // the CTA exits (bounded; the stages of the last STAGES k-tiles and
        // the low-rank tiles are the only ones that can still be in flight).
        for (int kt = max(0, num_kt - STAGES); kt < num_kt; ++kt)
          mbar_wait(full + kt % STAGES, (uint32_t)(kt / STAGES) & 1u, kDevErrTimeoutFull);
        if (RANK > 0) mbar_wait(lr_full, 0, kDevErrTimeoutFull);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_nvfp4(kGemmBM, kGemmBN);
      bool ok = true;
      for (int kt = 0; kt < num_kt && ok; ++kt) {
        const int s = kt % STAGES;
        const uint32_t ph = (uint32_t)(kt / STAGES) & 1u;
        if (!mbar_wait(full + s, ph, kDevErrTimeoutFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int kbs = min(kGemmKBPerStage, kb_total - kt * kGemmKBPerStage);
        unsigned char* st = smem + s * L::kStageBytes;
        const uint32_t sa = smem_u32(st);
        const uint32_t sb = sa + kTileABytes;
        const uint32_t sfa = sb + kTileBBytes;
        const uint32_t sfb = sfa + kGemmKBPerStage * kSfAtomBytes;
        for (int kb = 0; kb < kbs; ++kb) {
          tmem_cp_32x128b_x4(tmem + kTmemSfaCol + 4 * kb, smem_desc(sfa + kb * kSfAtomBytes, 16, 128, kSwizzleNone));
          tmem_cp_32x128b_x4(tmem + kTmemSfbCol + 4 * kb, smem_desc(sfb + kb * kSfAtomBytes, 16, 128, kSwizzleNone));
        }
        for (int kb = 0; kb < kbs; ++kb) {
          const uint64_t ad = smem_desc(sa + kb * 32, 16, 1024, kSwizzle128B);
          const uint64_t bd = smem_desc(sb + kb * 32, 16, 1024, kSwizzle128B);
          mma_nvfp4(tmem, ad, bd, idesc, tmem + kTmemSfaCol + 4 * kb, tmem + kTmemSfbCol + 4 * kb,
                    (kt | kb) != 0 ? 1u : 0u);
        }
        tc_commit(empty + s);   // stage s is free once these MMAs have read it
      }
      if (ok && RANK > 0) {
        if (mbar_wait(lr_full, 0, kDevErrTimeoutFull)) {
          tc_fence_after();
          const uint32_t idl = idesc_bf16(kGemmBM, kGemmBN);
          const uint32_t la = smem_u32(lr_a), lb = smem_u32(lr_b);
          for (int j = 0; j < RANK / 16; ++j) {
            const uint64_t ad = smem_desc(la + j * L::kLrSlabA, 16, 256, kSwizzle32B);
            const uint64_t bd = smem_desc(lb + j * L::kLrSlabB, 16, 256, kSwizzle32B);
            mma_bf16(tmem, ad, bd, idl, (num_kt > 0 || j > 0) ? 1u : 0u);
          }
        } else {
          ok = false;
        }
      }
      tc_commit(acc_full);   // arrives when every MMA above has completed
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const bool ok = mbar_wait(acc_full, 0, kDevErrTimeoutAccum);
    tc_fence_after();
    if (ok && !device_error_set()) {
      const int row = m0 + warp * 32 + lane;
      const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < kGemmBN; c += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(lane_addr + c, v);
        tmem_ld_wait();
        if (row < M) {
          uint32_t p[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
            p[i] = *reinterpret_cast<const uint32_t*>(&b);
          }
          uint4* dst = reinterpret_cast<uint4*>(Y + (size_t)row * N + n0 + c);
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[q] = make_uint4(p[4 * q], p[4 * q + 1], p[4 * q + 2], p[4 * q + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace svdq
