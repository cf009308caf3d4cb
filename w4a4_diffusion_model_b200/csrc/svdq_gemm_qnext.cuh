// The next layer's activation quantization, done in the GEMM epilogue.
//
// When a W4A4 layer feeds another one directly, its bf16 output Y is exactly
// the next layer's input X'. The next layer's smoothing and NVFP4 encoding
// (devpress.csdn.net SVDQuant walkthrough, eq. (1); the activation side of
// Fig. 6) can then run on the accumulator tile the epilogue already holds, so
// Y need not be written to memory and read back before it is quantized.
//
// Per epilogue warp (32 rows x 64*BOXES columns of one tile, row = lane), each
// thread encodes its row's 16-element groups from the packed bf16 registers
// with the quantizer's own recipe (smooth_group: x_hat = fp32(y * inv'); then
// encode_group_fast, two groups at a time, and encode_group_vals where a
// bracket straddles a midpoint: E4M3 scale of max|x_hat| / 6, E2M1 codes of
// x_hat / s, both of the exact quotients), writes the packed
// codes and the scale bytes in the native tile layout, and stores its band of
// Y (TMA, as the plain epilogue does) only when the caller asked for Y.
//
// With a next layer that has a low-rank branch (rank 16 or 32), the epilogue
// also forms that layer's down-projection T' = Y L1p'^T, which sums over all N
// columns, i.e. over every tile of a row: each tile's bf16 Y, staged in
// 128B-swizzled shared-memory boxes, is the A operand of tcgen05 bf16 pair
// MMAs against the tile's 256 columns of L1p' (TMA-loaded per tile), into a
// 32-column TMEM region; one epilogue thread of the even CTA issues them in a
// fixed order. The tile's fp32 partial of T' goes to the caller's workspace
// [N/256][M][rank'], and tprime_reduce_kernel adds the partials in tile order
// and rounds T' to bf16 (svdq_gemm_pair.cuh, svdq_api.cu).
#pragma once

#include <cuda_bf16.h>

#include "svdq_gemm_common.cuh"
#include "svdq_ptx.cuh"
#include "svdq_quant.cuh"
#include "svdq_quant_tma.cuh"

namespace svdq {

// The next layer's quantization inputs and outputs (device pointers).
struct NextQuant {
  const float* inv_lambda;        // [N] fp32 1/lambda' of the next layer
  uint8_t* qx;                    // [M][N/2] packed E2M1 codes
  uint8_t* sx;                    // native E4M3 scales of [ceil(M/128)*128][N/16]
  float* tp_ws;                   // [N/256][M][next_rank] fp32 partials of T' (next_rank > 0)
  int next_rank;                  // 0, 16 or 32
};

// The warp's inverse smoothing factors for columns col0 + [0, 128): lane l
// holds col0 + 4l .. 4l + 3. Loaded before the accumulator wait, so that the
// load's latency hides behind it; the encoder fetches a group's 16 factors
// from the four lanes that hold them.
__device__ __forceinline__ float4 epilogue_inv_factors(const NextQuant& nq, int col0, int lane) {
  return __ldg(reinterpret_cast<const float4*>(nq.inv_lambda + col0) + lane);
}

// One warp's band, quantized for the next layer from the packed bf16
// registers: packed codes and native scale words (32 rows x 64*BOXES columns,
// BOXES <= 2; inv4 from epilogue_inv_factors at col0).
template <int BOXES>
__device__ __forceinline__ void epilogue_encode_next(const uint32_t (&p)[32 * BOXES], const NextQuant& nq,
                                                     const float2* rcp_tbl, float4 inv4, int row0, int col0, int M,
                                                     int N, int lane) {
  static_assert(BOXES <= 2, "32 lanes x 4 factors cover 128 columns");
  const int row = row0 + lane;
  const int mpad = (M + 127) & ~127;
  const float2 six = recip_bracket(6.0f);
#pragma unroll
  for (int q = 0; q < BOXES; ++q) {   // four 16-groups (64 columns) at a time: one 32-bit word of scales
    uint32_t word = 0u;
#pragma unroll
    for (int j = 0; j < 4; j += 2) {   // two groups at a time (their common path interleaves)
      float4 l[2][4];
      float2 v[2][8];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int g = 4 * q + j + e;
#pragma unroll
        for (int k = 0; k < 4; ++k)   // factors 16g + 4k .. 16g + 4k + 3 sit in lane 4g + k
          l[e][k] = make_float4(__shfl_sync(0xFFFFFFFFu, inv4.x, 4 * g + k), __shfl_sync(0xFFFFFFFFu, inv4.y, 4 * g + k),
                                __shfl_sync(0xFFFFFFFFu, inv4.z, 4 * g + k), __shfl_sync(0xFFFFFFFFu, inv4.w, 4 * g + k));
        smooth_group(&p[8 * g], l[e], v[e]);
      }
      uint2 codes[2];
      uint32_t sb[2], bad = 0u;
      encode_group_fast(v[0], six, rcp_tbl, codes[0], sb[0], bad);
      encode_group_fast(v[1], six, rcp_tbl, codes[1], sb[1], bad);
      if (bad != 0u) {   // a midpoint inside some bracket: the exact recipe
        encode_group_vals(&p[8 * (4 * q + j)], l[0], rcp_tbl, codes[0], sb[0]);
        encode_group_vals(&p[8 * (4 * q + j + 1)], l[1], rcp_tbl, codes[1], sb[1]);
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int g = 4 * q + j + e;
        if (row < M)
          *reinterpret_cast<uint2*>(nq.qx + (size_t)row * (size_t)(N >> 1) + ((col0 + 16 * g) >> 1)) = codes[e];
        word |= sb[e] << (8 * (j + e));
      }
    }
    // rows past M carry zero accumulators, hence the zero scales of the padding rows
    if (row < mpad) *reinterpret_cast<uint32_t*>(nq.sx + native_scale_offset(row, (col0 >> 4) + 4 * q, N)) = word;
  }
}

// Epilogue of one warp: quantize its band for the next layer, then store the
// band of Y if asked (through the warp's 128B-swizzled staging box).
template <int BOXES>
__device__ __forceinline__ void epilogue_quantize_next(const uint32_t (&p)[32 * BOXES], unsigned char* box,
                                                       const NextQuant& nq, const float2* rcp_tbl, float4 inv4,
                                                       const void* tm_y, bool store_y, int row0, int col0, int M,
                                                       int N, int lane) {
  epilogue_encode_next<BOXES>(p, nq, rcp_tbl, inv4, row0, col0, M, N, lane);
  if (store_y) epilogue_store_band<BOXES>(p, box, tm_y, col0, row0, lane, row0 < M);
}

// Write box b (64 columns) of a warp's band into its 128B-swizzled staging
// box: row `lane`, 16-byte chunk c at (c ^ (lane & 7)).
__device__ __forceinline__ void epilogue_stage_box(const uint32_t* p, unsigned char* box, int lane) {
  const uint32_t box_addr = smem_u32(box);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint32_t addr = box_addr + lane * 128 + ((c ^ (lane & 7)) << 4);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(p[4 * c]), "r"(p[4 * c + 1]),
                 "r"(p[4 * c + 2]), "r"(p[4 * c + 3])
                 : "memory");
  }
}

// T' = sum over the N/256 column tiles of their fp32 partials, in tile order,
// rounded to bf16: ws [slices][M][r], T [M][r]. Four outputs per thread.
__global__ void __launch_bounds__(256) tprime_reduce_kernel(const float4* __restrict__ ws,
                                                            __nv_bfloat16* __restrict__ T, long long n4,
                                                            int slices) {
  grid_dependency_wait();     // the GEMM that wrote the partials is complete
  grid_launch_dependents();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  float4 s = ws[i];
  for (int t = 1; t < slices; ++t) {
    const float4 v = ws[(long long)t * n4 + i];
    s.x = __fadd_rn(s.x, v.x);
    s.y = __fadd_rn(s.y, v.y);
    s.z = __fadd_rn(s.z, v.z);
    s.w = __fadd_rn(s.w, v.w);
  }
  const __nv_bfloat162 lo = __floats2bfloat162_rn(s.x, s.y), hi = __floats2bfloat162_rn(s.z, s.w);
  reinterpret_cast<uint2*>(T)[i] = make_uint2(*reinterpret_cast<const uint32_t*>(&lo),
                                              *reinterpret_cast<const uint32_t*>(&hi));
}

}  // namespace svdq
