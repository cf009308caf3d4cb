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
// with the quantizer's own recipe (encode_group_bf16: x_hat = fp32(y * inv'),
// E4M3 scale of max|x_hat| / 6, E2M1 codes of x_hat / s), writes the packed
// codes and the scale bytes in the native tile layout, and stores its band of
// Y (TMA, as the plain epilogue does) only when the caller asked for Y.
//
// The next layer's low-rank down-projection T' = Y L1p'^T is not formed here:
// it sums over all N, i.e. over every tile of a row, and on this kernel it
// would have to run either as warp-level MMAs, which wait for the tcgen05 MMAs
// of the running mainloop (measured: +46 us on the FLUX MLP-up projection for
// a rank of 16), or as tcgen05 MMAs, for whose operands the 256 x 256 pair
// tiles leave no shared or tensor memory. A next layer with a low-rank branch
// therefore goes through Y and the quantizer (svdq_api.cu).
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
};

// Epilogue of one warp: quantize its band for the next layer, then store the
// band of Y if asked (through the warp's 128B-swizzled staging box).
template <int BOXES>
__device__ __forceinline__ void epilogue_quantize_next(const uint32_t (&p)[32 * BOXES], unsigned char* box,
                                                       const NextQuant& nq, const float2* rcp_tbl, const void* tm_y,
                                                       bool store_y, int row0, int col0, int M, int N, int lane) {
  const int row = row0 + lane;
  const int mpad = (M + 127) & ~127;
#pragma unroll
  for (int q = 0; q < BOXES; ++q) {   // four 16-groups (64 columns) at a time: one 32-bit word of scales
    uint32_t word = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int g = 4 * q + j;
      uint2 codes;
      uint32_t sb;
      encode_group_bf16(&p[8 * g], nq.inv_lambda + col0 + 16 * g, rcp_tbl, codes, sb);
      if (row < M) *reinterpret_cast<uint2*>(nq.qx + (size_t)row * (size_t)(N >> 1) + ((col0 + 16 * g) >> 1)) = codes;
      word |= sb << (8 * j);
    }
    // rows past M carry zero accumulators, hence the zero scales of the padding rows
    if (row < mpad) *reinterpret_cast<uint32_t*>(nq.sx + native_scale_offset(row, (col0 >> 4) + 4 * q, N)) = word;
  }
  if (store_y) epilogue_store_band<BOXES>(p, box, tm_y, col0, row0, lane, row0 < M);
}

}  // namespace svdq
