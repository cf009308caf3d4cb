// DeltaQuant-style core + delta encoding of video activations (libaedu.com
// article on 4-bit diffusion-model quantization, DeltaQuant paragraphs: the
// tokens of a local 3-D spatio-temporal block share a core token, their mean,
// kept in FP8; each token's difference to it is quantized to 4 bits).
//
// Tokens are rows of X [F*H*W][C] bf16 in frame, row, column order; blocks are
// 2 x 2 x 2 tokens tiled from the origin, edge blocks holding the tokens that
// exist (n = 1, 2, 4 or 8 of them). Per block b and channel c:
//   core[b][c] = E4M3_RNE_satfinite(sum / n) of the exact sum of the block's
//                tokens, rounded once; a negative mean rounding to zero keeps
//                the sign bit, a zero sum encodes +0;
//   delta[t][c] = fp32(x[t][c] - decode(core[b][c])), the exact difference
//                rounded once (one fp32 subtraction: both operands are fp32
//                values), NVFP4-encoded along C with the library's codec
//                (nvfp4_encode16: E4M3 scale of amax / 6, E2M1 codes of the
//                exact quotients), codes packed two per byte, scales in the
//                native tile layout of the 4-bit GEMM.
//
// The exact sum. Eight bf16 values carry 8-bit significands; when the nonzero
// ones span at most 13 binades (max|x| <= 2^13 min|x|) their sum needs at most
// 8 + 13 + 3 = 24 bits and the fp32 additions are exact, and so is the mean
// (n is a power of two): the hardware fp32 -> E4M3 conversion then rounds the
// exact mean once. A channel whose values span more binades (or whose values
// reach 2^124, where eight of them could overflow fp32) takes the fp64 path:
// the sum in token order, exact for spreads up to ~45 binades and otherwise
// the same fp64 additions the reference makes, rounded to E4M3 from fp64.
//
// A CTA of 128 threads handles one block and up to 64 16-channel groups
// (grid: x = block, y = 1024-channel chunk); two lanes share a group, 8
// channels each, so that a warp reads each token row as one coalesced 512-byte
// span. A lane forms its 8 sums and cores, then encodes each token's deltas
// with the pair recipe nvfp4_encode8_pair (which resolves midpoint ties one
// element at a time: they are common in deltas); the 8 lanes of 4 consecutive
// groups pool their scale bytes into one 32-bit store. Rows of the last 128-row scale
// atom past the last token are zeroed by the host before the launch.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "svdq_quant.cuh"

namespace svdq {

__device__ __forceinline__ float e4m3_to_float(uint32_t byte) {
  return __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)byte, __NV_E4M3)));
}

// The two bf16 values of w (low half first) plus, or minus, fp32 operands:
// exact conversions, one round-to-nearest-even each (mixed-precision
// add / sub with the bf16 operand first).
__device__ __forceinline__ float2 bf16x2_add_f32(uint32_t w, float2 c) {
  float2 r;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "add.rn.f32.bf16 %0, l, %3;\n\tadd.rn.f32.bf16 %1, h, %4;\n\t}"
      : "=f"(r.x), "=f"(r.y) : "r"(w), "f"(c.x), "f"(c.y));
  return r;
}

__device__ __forceinline__ float2 bf16x2_sub_f32(uint32_t w, float c0, float c1) {
  float2 r;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "sub.rn.f32.bf16 %0, l, %3;\n\tsub.rn.f32.bf16 %1, h, %4;\n\t}"
      : "=f"(r.x), "=f"(r.y) : "r"(w), "f"(c0), "f"(c1));
  return r;
}

// Per 16-bit half: max and min of unsigned values.
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ uint32_t min_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

constexpr int kDqThreads = 128;
constexpr int kDqGroupsPerCta = kDqThreads / 2;
// Six CTAs per SM (79 registers a thread, no spill): the kernel is bound by
// issue latency, and more resident warps hide more of it (measured 1880
// against 1851 GB/s at five CTAs; seven and eight spill and run at ~1860).

__global__ void __launch_bounds__(kDqThreads, 6) deltaquant_encode_kernel(const __nv_bfloat16* __restrict__ X,
                                                                       uint8_t* __restrict__ core,
                                                                       uint8_t* __restrict__ Qd,
                                                                       uint8_t* __restrict__ Sd, int F, int H, int W,
                                                                       int C) {
  __shared__ float2 rcp_tbl[128];                         // bracket of 1/s per E4M3 scale byte (sign clear)
  rcp_tbl[threadIdx.x] = e4m3_recip_bracket(threadIdx.x);
  const int G = C >> 4;                                   // 16-channel groups per token (a multiple of 4)
  const int nbh = (H + 1) >> 1, nbw = (W + 1) >> 1;
  const int b = blockIdx.x;                               // the block
  const int bw = b % nbw, bh = (b / nbw) % nbh, bf = b / (nbw * nbh);
  const int gl = blockIdx.y * kDqGroupsPerCta + (threadIdx.x >> 1);
  const bool live = gl < G;                               // lanes past C (whole quads of groups) store nothing
  const int g = live ? gl : G - 4 + ((threadIdx.x >> 1) & 3);
  const int half = threadIdx.x & 1;
  const int c0 = 16 * g + 8 * half;                       // this lane's 8 channels

  // the block's tokens in token order (frame, row, column)
  int rows[8];
  int n = 0, present = 0;
#pragma unroll
  for (int df = 0; df < 2; ++df)
#pragma unroll
    for (int dh = 0; dh < 2; ++dh)
#pragma unroll
      for (int dw = 0; dw < 2; ++dw) {
        const int f = 2 * bf + df, h = 2 * bh + dh, w = 2 * bw + dw;
        const int t = 4 * df + 2 * dh + dw;
        const bool ok = f < F && h < H && w < W;
        rows[t] = ok ? (f * H + h) * W + w : -1;
        n += ok;
        present |= ok ? 1 << t : 0;
      }
  uint32_t xw[32];                                        // token t, pair i at xw[4 t + i]
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    uint4 a = make_uint4(0u, 0u, 0u, 0u);
    if (rows[t] >= 0) a = __ldg(reinterpret_cast<const uint4*>(X + (size_t)rows[t] * C + c0));
    xw[4 * t + 0] = a.x; xw[4 * t + 1] = a.y; xw[4 * t + 2] = a.z; xw[4 * t + 3] = a.w;
  }
  // fp32 sums (exact when the spread test below passes), |x| max and nonzero
  // |x| min per channel, the last two on the bf16 bit patterns of a channel
  // pair at once (magnitudes order like their patterns; a zero becomes 0x7FFF
  // through a borrow-free per-half decrement, above every finite magnitude
  // minus one); missing tokens hold +0 and change none of them
  float2 sum[4];
  uint32_t mx2[4], mn2[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    sum[i] = make_float2(0.f, 0.f);
    mx2[i] = 0u;
    mn2[i] = 0x7FFF7FFFu;
  }
#pragma unroll
  for (int t = 0; t < 8; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t w = xw[4 * t + i];
      sum[i] = bf16x2_add_f32(w, sum[i]);
      mx2[i] = max_u16x2(mx2[i], w & 0x7FFF7FFFu);
      mn2[i] = min_u16x2(mn2[i], ((w | 0x80008000u) - 0x00010001u) & 0x7FFF7FFFu);
    }
  const float inv_n = 1.0f / (float)n;                    // n is 1, 2, 4 or 8: exact
  float cval[8];
  uint32_t cb[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t mxb = (mx2[i >> 1] >> (16 * (i & 1))) & 0xFFFFu;   // max |x|, bf16 bits
    const uint32_t mnz = (mn2[i >> 1] >> (16 * (i & 1))) & 0xFFFFu;   // min nonzero |x| bits - 1, 0x7FFF: none
    const float mxf = __uint_as_float(mxb << 16), mnf = __uint_as_float((mnz + 1u) << 16);
    const bool exact = mxb < 0x7D80u && (mnz == 0x7FFFu || mxf <= mnf * 8192.0f);   // 0x7D80: 2^124
    uint32_t byte;
    if (exact) {
      const float mean = ((i & 1) ? sum[i >> 1].y : sum[i >> 1].x) * inv_n;
      byte = mean == 0.f ? 0u : (uint32_t)__nv_cvt_float_to_fp8(mean, __NV_SATFINITE, __NV_E4M3);
    } else {   // wide range: the fp64 sum in token order (i and t are compile-time: registers only)
      double sd = 0.0;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (!(present & (1 << t))) continue;
        const uint32_t w = xw[4 * t + (i >> 1)];
        sd += (double)((i & 1) ? bf16hi(w) : bf16lo(w));
      }
      byte = sd == 0.0 ? 0u : (uint32_t)__nv_cvt_double_to_fp8(sd / (double)n, __NV_SATFINITE, __NV_E4M3);
    }
    cval[i] = e4m3_to_float(byte);
    cb[i >> 2] |= byte << (8 * (i & 3));
  }
  if (live) *reinterpret_cast<uint2*>(core + (size_t)b * C + c0) = make_uint2(cb[0], cb[1]);

  // Every lane runs all eight token positions (edge blocks lack some tokens):
  // the shuffles are taken by the whole warp, only the stores depend on the
  // token existing.
  const int lane = threadIdx.x & 31;
  const float2 six = recip_bracket(6.0f);
  __syncthreads();                                        // the reciprocal table is complete
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    float2 d[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) d[i] = bf16x2_sub_f32(xw[4 * t + i], cval[2 * i], cval[2 * i + 1]);
    uint32_t codes, sb;
    nvfp4_encode8_pair(d, rcp_tbl, six, codes, sb);
    // lanes 8j, 8j+2, 8j+4, 8j+6 hold the scales of groups 4j'..4j'+3
    const uint32_t s1 = __shfl_sync(0xFFFFFFFFu, sb, (lane + 2) & 31), s2 = __shfl_sync(0xFFFFFFFFu, sb, (lane + 4) & 31),
                   s3 = __shfl_sync(0xFFFFFFFFu, sb, (lane + 6) & 31);
    if (!live || rows[t] < 0) continue;
    const size_t row = (size_t)rows[t];
    *reinterpret_cast<uint32_t*>(Qd + row * (size_t)(C >> 1) + (c0 >> 1)) = codes;
    if ((lane & 7) == 0)
      *reinterpret_cast<uint32_t*>(Sd + native_scale_offset(rows[t], g, C)) = sb | (s1 << 8) | (s2 << 16) | (s3 << 24);
  }
}

}  // namespace svdq
