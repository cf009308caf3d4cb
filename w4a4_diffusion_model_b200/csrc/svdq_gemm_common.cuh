// Pieces shared by the two W4A4 GEMM kernels (single CTA and CTA pair):
// tile constants, the TMEM column plan, the scale-warp routine that moves
// block scales from shared memory into TMEM, and the epilogue.
//
// Why scale warps: tcgen05.cp would copy the scale atoms inside the tensor
// pipe, in order with the MMAs, and any later shared-memory access by the
// issuing thread waits for those copies; the MMA issuer would then idle for a
// large part of every k-tile. Instead four warps (one per TMEM lane quadrant)
// load each k-tile's scale atoms from shared memory and write them with
// tcgen05.st into the TMEM scale buffer of the item's ring stage, and the MMA
// issuer only ever waits for "scales ready" and "accumulator free".
#pragma once

#include <cuda_bf16.h>

#include "svdq_ptx.cuh"

namespace svdq {

constexpr int kGemmBKBytes = 128;                 // 256 FP4 elements per k-tile row (128B swizzle)
constexpr int kGemmKBPerStage = 4;                // 64-element MMA K blocks per k-tile
constexpr int kGemmLrK = 64;                      // bf16 K elements per low-rank k-tile
constexpr int kSfAtomBytes = 512;                 // 128 rows x 4 scales (one MMA K block)

// Warp roles: 0..7 epilogue, 8 producer, 9 MMA issuer / TMEM allocator, 10..13 scale warps.
constexpr int kGemmEpiWarps = 8;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kSfWarp0 = 10;
constexpr int kSfWarps = 4;
// 14 warps: one SM sub-partition (16384 registers) holds 4 of them, so a
// thread may use at most 128 registers.
constexpr int kGemmThreads = 32 * (kGemmEpiWarps + 2 + kSfWarps);

// TMEM: accumulator columns [0, 256); then one scale buffer of 48 columns per
// ring stage (A scales: 4 columns per K block, then B scales: 8 per K block),
// so that the one tcgen05.commit that frees a ring stage also frees its scale
// buffer. At most 5 stages fit: 256 + 5 * 48 = 496 <= 512 columns.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = 256;
constexpr uint32_t kSfBufCols = 4 * kGemmKBPerStage + 8 * kGemmKBPerStage;
constexpr int kMaxSfBufs = (int)((kTmemCols - kAccCols) / kSfBufCols);
__host__ __device__ constexpr uint32_t sf_buf_col(int b) { return kAccCols + (uint32_t)b * kSfBufCols; }

// Epilogue staging: one 32-row x 64-column bf16 box (4 KB) per epilogue warp.
constexpr int kEpiBoxCols = 64;
constexpr int kEpiBoxBytes = 32 * kEpiBoxCols * 2;

// Scale warp `q` (lane quadrant) writes one k-tile's scales into the TMEM
// buffer at column `col`, lanes 32q..32q+31:
//   A: column 4*kb + j of lane 32q+i  <-  byte word j of line i of A atom kb
//      (the MMA reads column 4*kb + q at lane 32q+i: the scales of A row 32q+i)
//   B: column 8*kb + c of lane 32q+i  <-  scales of B row 32c+i, i.e. word c of
//      line i of B atom kb (c < 4) or of the second 128-row half (c >= 4)
// which is the layout tcgen05.cp.32x128b.warpx4 would produce. With a third
// 128-row block of B (`sfb2`, for a second MMA of N = 128), its scales follow
// at column 48 + 4*kb + c, laid out like A's.
__device__ __forceinline__ void scales_to_tmem(uint32_t tmem, int q, int lane, const unsigned char* sfa,
                                               const unsigned char* sfb0, const unsigned char* sfb1, uint32_t col,
                                               const unsigned char* sfb2 = nullptr) {
  uint32_t ra[16], rb[32];
#pragma unroll
  for (int kb = 0; kb < kGemmKBPerStage; ++kb) {
    const uint4 a = *reinterpret_cast<const uint4*>(sfa + kb * kSfAtomBytes + lane * 16);
    ra[4 * kb] = a.x; ra[4 * kb + 1] = a.y; ra[4 * kb + 2] = a.z; ra[4 * kb + 3] = a.w;
    const uint4 b0 = *reinterpret_cast<const uint4*>(sfb0 + kb * kSfAtomBytes + lane * 16);
    const uint4 b1 = *reinterpret_cast<const uint4*>(sfb1 + kb * kSfAtomBytes + lane * 16);
    rb[8 * kb] = b0.x; rb[8 * kb + 1] = b0.y; rb[8 * kb + 2] = b0.z; rb[8 * kb + 3] = b0.w;
    rb[8 * kb + 4] = b1.x; rb[8 * kb + 5] = b1.y; rb[8 * kb + 6] = b1.z; rb[8 * kb + 7] = b1.w;
  }
  const uint32_t t = tmem + ((uint32_t)(q * 32) << 16) + col;
  tmem_st_32x32b_x16(t, ra);
  tmem_st_32x32b_x32(t + 4 * kGemmKBPerStage, rb);
  if (sfb2 != nullptr) {
#pragma unroll
    for (int kb = 0; kb < kGemmKBPerStage; ++kb) {
      const uint4 b2 = *reinterpret_cast<const uint4*>(sfb2 + kb * kSfAtomBytes + lane * 16);
      ra[4 * kb] = b2.x; ra[4 * kb + 1] = b2.y; ra[4 * kb + 2] = b2.z; ra[4 * kb + 3] = b2.w;
    }
    tmem_st_32x32b_x16(t + 12 * kGemmKBPerStage, ra);
  }
}

// Drain 32 * CHUNKS accumulator columns of this warp's lane band (32 at a
// time) and pack them to bf16 pairs: p[j] holds columns 2j and 2j+1.
template <int CHUNKS>
__device__ __forceinline__ void epilogue_drain_pack(uint32_t taddr, uint32_t (&p)[16 * CHUNKS]) {
#pragma unroll
  for (int c = 0; c < CHUNKS; ++c) {
    uint32_t v[32];
    tmem_ld_32x32b_x32(taddr + 32 * c, v);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const __nv_bfloat162 bb = __floats2bfloat162_rn(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
      p[16 * c + i] = *reinterpret_cast<const uint32_t*>(&bb);
    }
  }
}

// Write one warp's 32 x (64 * BOXES) bf16 band (row `lane` = p) as 32 x 64
// boxes through a 128B-swizzled staging box and TMA stores (clipped at the edge).
template <int BOXES>
__device__ __forceinline__ void epilogue_store_band(const uint32_t (&p)[32 * BOXES], unsigned char* box,
                                                    const void* tm_y, int col0, int row0, int lane, bool store) {
  const uint32_t box_addr = smem_u32(box);
#pragma unroll
  for (int b = 0; b < BOXES; ++b) {
    if (lane == 0) bulk_wait_read<0>();   // the previous store from this box has read it
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      // row `lane`: 16-byte chunk c at (c ^ (lane & 7)) -- the 128B swizzle pattern
      const uint32_t addr = box_addr + lane * 128 + ((c ^ (lane & 7)) << 4);
      const int e = 32 * b + 4 * c;
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(p[e]), "r"(p[e + 1]), "r"(p[e + 2]),
                   "r"(p[e + 3])
                   : "memory");
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && store) {
      tma_store_2d_evict_first(tm_y, box, col0 + 64 * b, row0);   // Y is not read again here
      bulk_commit();
    }
  }
}

}  // namespace svdq
