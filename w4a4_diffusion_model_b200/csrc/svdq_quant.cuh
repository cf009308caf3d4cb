// Activation-side helpers of the SVDQuant W4A4 layer (the quantization kernel
// itself is quantize_tma_kernel):
//   * nvfp4_encode16: the NVFP4 group recipe (also used for the weights);
//   * channel_amax_kernel: per-channel max|x| (handbook SmoothQuant section);
//   * scales_native_to_canonical_kernel: inspection helper;
//   * lowrank_up_rmw_kernel: the unfused up-projection.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "svdq_ptx.cuh"

namespace svdq {

// Byte offset of scale (row r, 16-group g) in the native tile layout
// (128-row x 64-element atoms of 512 bytes; see include/svdq.h).
__host__ __device__ __forceinline__ size_t native_scale_offset(int r, int g, int K) {
  const int kb = g >> 2, j = g & 3;
  const int rb = r >> 7, rr = r & 127;
  return ((size_t)rb * (size_t)(K >> 6) + (size_t)kb) * 512u + 16u * (rr & 31) + 4u * (rr >> 5) + j;
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two IEEE round-to-nearest fp32 products in one instruction.
__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// max(|a|, |b|, |c|).
__device__ __forceinline__ float max3_abs(float a, float b, float c) {
  float d;
  asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// E2M1 codes (round to nearest even, saturating) of 4 value pairs times f,
// packed into one word: element 2i in the low nibble of byte i.
__device__ __forceinline__ uint32_t e2m1_word(const float2* v, float f) {
  const float2 p0 = mul2_rn(v[0], make_float2(f, f)), p1 = mul2_rn(v[1], make_float2(f, f));
  const float2 p2 = mul2_rn(v[2], make_float2(f, f)), p3 = mul2_rn(v[3], make_float2(f, f));
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(p0.x), "f"(p0.y), "f"(p1.x), "f"(p1.y), "f"(p2.x), "f"(p2.y), "f"(p3.x), "f"(p3.y));
  return r;
}

// ---------------------------------------------------------------- exact-quotient rounding
// The codes are round-to-nearest-even images of the EXACT quotient v / s
// (walkthrough eq. (1): round(X / s)). Multiplying by one rounded reciprocal
// would not do: it carries up to two fp32 roundings and picks the wrong code
// when v / s sits on or next to a midpoint of the code grid. Instead each
// value is multiplied by two reciprocals that bracket 1 / s,
//   r = fp32(1/s),  lo = fp32(r (1 - 2^-21)),  hi = fp32(r (1 + 2^-21)),
// for which lo < (1/s)(1 - 2^-22) and hi > (1/s)(1 + 2^-22) (each step errs by
// at most 2^-24 relative), hence |fp32(v lo)| < |v / s| < |fp32(v hi)| for
// every fp32 v. Rounding is monotone, so when both products give the same
// code that code is the exact one. They differ only when a midpoint lies in
// the bracket (relative width < 2^-19.9, so at most one midpoint, and the two
// codes are neighbours); then |v| is compared with the midpoint above the
// lower code, times s, which is exact in fp32 (midpoints carry at most 4
// significant bits, scales at most 11), and a tie goes to the even code.
__device__ __forceinline__ float2 recip_bracket(float s) {
  const float r = __frcp_rn(s);
  return make_float2(__fmul_rn(r, 1.0f - 0x1p-21f), __fmul_rn(r, 1.0f + 0x1p-21f));
}

// Entry `byte` of the table of bracketing reciprocals indexed by an E4M3
// scale byte with the sign bit clear: recip_bracket of its value, and (0, 0)
// for byte 0 (a zero scale: encode_group_fast multiplies by zero and selects
// +0 codes; encode_group_vals never looks it up).
__device__ __forceinline__ float2 e4m3_recip_bracket(uint32_t byte) {
  if (byte == 0u) return make_float2(0.f, 0.f);
  const float sv = __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)byte, __NV_E4M3)));
  return recip_bracket(sv);
}

// The exact code of v / s, given the code a of the lower bracket product
// v lo (sign bit included; the code of v hi is a or its upper neighbour):
// compare |v| with the midpoint above a's magnitude m, times s (exact in fp32:
// 4 x midpoint, looked up as a byte -- 1, 3, 5, 7, 10, 14, 20 for m = 0..6,
// 255 for m = 7, where nothing lies above -- times s / 4). Above it: m + 1;
// on it: the even one of m, m + 1; below it: m. Branch-free, so that a warp
// whose lanes need it for different elements runs it once.
__device__ __forceinline__ uint32_t e2m1_exact_nibble(float v, float s4, uint32_t a) {
  const uint32_t m = a & 7u;
  const float t = __fmul_rn((float)(__byte_perm(0x07050301u, 0xFF140E0Au, m) & 0xFFu), s4);   // exact
  const float x = fabsf(v);
  const uint32_t up = (x > t || (x == t && (m & 1u))) ? 1u : 0u;
  return (m + up) | (a & 8u);
}

// E2M1 byte (element 2i low, 2i+1 high) of a pair scaled by `inv`.
__device__ __forceinline__ uint32_t e2m1_pair(float2 v, float inv) {
  return (uint32_t)__nv_cvt_float2_to_fp4x2(make_float2(__fmul_rn(v.x, inv), __fmul_rn(v.y, inv)), __NV_E2M1,
                                            cudaRoundNearest) & 0xFFu;
}

// Packed codes of 8 pairs (16 values, one NVFP4 group) given the codes of the
// two bracket products (`lo`, `hi`; pair i in byte i % 4 of word i / 4): when
// they differ anywhere, every element is recomputed exactly from `lo` (for an
// element whose bracket holds no midpoint the recomputation returns its code).
__device__ __forceinline__ uint2 e2m1_group_exact(const float2 (&v)[8], float s, uint2 lo, uint2 hi) {
  if (((lo.x ^ hi.x) | (lo.y ^ hi.y)) == 0u) return lo;
  const float s4 = 0.25f * s;
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t a = ((i < 4 ? lo.x : lo.y) >> (8 * (i & 3))) & 0xFFu;
    const uint32_t byte = e2m1_exact_nibble(v[i].x, s4, a & 15u) | (e2m1_exact_nibble(v[i].y, s4, a >> 4) << 4);
    w[i >> 2] |= byte << (8 * (i & 3));
  }
  return make_uint2(w[0], w[1]);
}

// NVFP4 encoding of 16 fp32 values (one group):
//   s = E4M3_rne_satfinite(fp32(max|v| / 6)) (fp32 division then RNE equals
//   one rounding of the exact quotient: a midpoint times 6 is exact in fp32);
//   q_i = E2M1_rne_satfinite(v_i / s) of the exact quotient; all codes +0 when
//   s decodes to 0. Element 2i lands in the low nibble of byte i.
__device__ __forceinline__ void nvfp4_encode16(const float (&v)[16], uint2& codes, uint32_t& sbyte) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const float s32 = __fdiv_rn(amax, 6.0f);
  const __nv_fp8_storage_t sb = __nv_cvt_float_to_fp8(s32, __NV_SATFINITE, __NV_E4M3);
  const float sval = __half2float(__half(__nv_cvt_fp8_to_halfraw(sb, __NV_E4M3)));
  sbyte = (uint32_t)sb;
  if (sval == 0.f) {
    codes = make_uint2(0u, 0u);
    return;
  }
  const float2 ib = recip_bracket(sval);
  float2 p[8];
  uint32_t lo[2] = {0u, 0u}, hi[2] = {0u, 0u};
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    p[b] = make_float2(v[2 * b], v[2 * b + 1]);
    lo[b >> 2] |= e2m1_pair(p[b], ib.x) << (8 * (b & 3));
    hi[b >> 2] |= e2m1_pair(p[b], ib.y) << (8 * (b & 3));
  }
  codes = e2m1_group_exact(p, sval, make_uint2(lo[0], lo[1]), make_uint2(hi[0], hi[1]));
}

// The same NVFP4 recipe for a group of 16 held by two lanes (lane ^ 1), 8
// values each (element 2i in d[i].x, 2i+1 in d[i].y): the group's amax is
// pooled with one shuffle, both lanes derive the same scale, and each lane
// returns the packed codes of its own 8 values (one 32-bit word: element j in
// nibble j). Made for inputs on which exact midpoint ties are common (the
// DeltaQuant deltas: a bf16 token minus an E4M3 core, divided by an E4M3
// scale, lands on a midpoint for ~2 % of elements):
//   scale byte: amax times the bracket of 1/6, both products converted by one
//   cvt; the IEEE quotient only where the two bytes differ;
//   codes: both bracket products of 1/s (rcp_tbl: e4m3_recip_bracket per byte);
//   each nibble where they differ is resolved on its own by e2m1_exact_nibble,
//   looping over the differing nibbles only.
// Every lane of the warp must call it.
__device__ __forceinline__ void nvfp4_encode8_pair(const float2 (&d)[4], const float2* rcp_tbl, float2 six,
                                                   uint32_t& codes, uint32_t& sbyte) {
  const float m = fmaxf(max3_abs(d[0].x, d[0].y, d[1].x), max3_abs(d[1].y, d[2].x, max3_abs(d[2].y, d[3].x, d[3].y)));
  const float amax = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
  const uint32_t two = (uint32_t)__nv_cvt_float2_to_fp8x2(mul2_rn(make_float2(amax, amax), six), __NV_SATFINITE,
                                                          __NV_E4M3);
  uint32_t b = two & 0xFFu;
  if ((two >> 8) != b) b = (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(amax, 6.0f), __NV_SATFINITE, __NV_E4M3);
  sbyte = b;
  const float2 ib = rcp_tbl[b & 0x7Fu];
  uint32_t lo = e2m1_word(d, ib.x);
  uint32_t diff = lo ^ e2m1_word(d, ib.y);
  if (diff != 0u) {
    const float s4 = 0.25f * __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)b, __NV_E4M3)));
    do {
      const int j = (__ffs((int)diff) - 1) >> 2;     // the lowest differing element
      float v = d[0].x;
      v = j == 1 ? d[0].y : v;
      v = j == 2 ? d[1].x : v;
      v = j == 3 ? d[1].y : v;
      v = j == 4 ? d[2].x : v;
      v = j == 5 ? d[2].y : v;
      v = j == 6 ? d[3].x : v;
      v = j == 7 ? d[3].y : v;
      const uint32_t sh = 4u * (uint32_t)j;
      const uint32_t nib = e2m1_exact_nibble(v, s4, (lo >> sh) & 0xFu);
      lo = (lo & ~(0xFu << sh)) | (nib << sh);
      diff &= ~(0xFu << sh);
    } while (diff != 0u);
  }
  codes = b != 0u ? lo : 0u;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// amax[j] = max_m |X[m][j]| over bf16 X [M][K]; amax must be zeroed first.
// Each thread owns 8 adjacent columns and a strided set of rows; non-negative
// floats order like their bit patterns, so an integer atomicMax is exact.
__global__ void channel_amax_kernel(const __nv_bfloat16* __restrict__ X, float* __restrict__ amax, int M, int K,
                                    int rows_per_block) {
  const int col8 = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (col8 >= K) return;
  const int r0 = blockIdx.y * rows_per_block;
  const int r1 = min(M, r0 + rows_per_block);
  float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int r = r0; r < r1; ++r) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(X + (size_t)r * K + col8));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      m[2 * i] = fmaxf(m[2 * i], fabsf(bf16lo(w[i])));
      m[2 * i + 1] = fmaxf(m[2 * i + 1], fabsf(bf16hi(w[i])));
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i)
    atomicMax(reinterpret_cast<unsigned int*>(amax) + col8 + i, __float_as_uint(m[i]));
}

__global__ void scales_native_to_canonical_kernel(const uint8_t* __restrict__ native, uint8_t* __restrict__ canon,
                                                  int rows, int K) {
  const int G = K >> 4;
  const size_t n = (size_t)rows * G;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(i / G), g = (int)(i % G);
    canon[i] = native[native_scale_offset(r, g, K)];
  }
}

// Unfused up-projection: Y = bf16(fp32(Y) + T L2t^T). A CTA (4 warps) owns a
// 64 x 128 tile of Y; T and L2t tiles are staged in shared memory, each warp
// computes 16 rows x 128 columns with mma.sync, the fp32 results go through
// shared memory so that Y is read and written with coalesced 16-byte accesses.
template <int RANK>
__global__ void __launch_bounds__(128) lowrank_up_rmw_kernel(const __nv_bfloat16* __restrict__ T,
                                                             const __nv_bfloat16* __restrict__ L2t,
                                                             __nv_bfloat16* __restrict__ Y, int M, int N) {
  constexpr int BM = 64, BN = 128, LDS = RANK + 8;   // +8 bf16 pads rows against bank conflicts
  extern __shared__ __align__(16) unsigned char up_smem[];
  __nv_bfloat16* Ts = reinterpret_cast<__nv_bfloat16*>(up_smem);
  __nv_bfloat16* Ls = Ts + BM * LDS;
  float* Ys = reinterpret_cast<float*>(up_smem);      // reused after the MMAs: [BM][BN]
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;

  for (int i = threadIdx.x; i < BM * RANK / 8; i += 128) {
    const int r = i / (RANK / 8), c = (i % (RANK / 8)) * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (m0 + r < M) v = __ldg(reinterpret_cast<const uint4*>(T + (size_t)(m0 + r) * RANK + c));
    *reinterpret_cast<uint4*>(Ts + r * LDS + c) = v;
  }
  for (int i = threadIdx.x; i < BN * RANK / 8; i += 128) {
    const int r = i / (RANK / 8), c = (i % (RANK / 8)) * 8;
    *reinterpret_cast<uint4*>(Ls + r * LDS + c) =
        __ldg(reinterpret_cast<const uint4*>(L2t + (size_t)(n0 + r) * RANK + c));
  }
  __syncthreads();

  float acc[BN / 8][4];
#pragma unroll
  for (int i = 0; i < BN / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  const __nv_bfloat16* Tw = Ts + warp * 16 * LDS;
#pragma unroll
  for (int ks = 0; ks < RANK / 16; ++ks) {
    const int k = ks * 16 + 2 * t;
    const uint32_t a0 = *reinterpret_cast<const uint32_t*>(Tw + g * LDS + k);
    const uint32_t a1 = *reinterpret_cast<const uint32_t*>(Tw + (g + 8) * LDS + k);
    const uint32_t a2 = *reinterpret_cast<const uint32_t*>(Tw + g * LDS + k + 8);
    const uint32_t a3 = *reinterpret_cast<const uint32_t*>(Tw + (g + 8) * LDS + k + 8);
#pragma unroll
    for (int nt = 0; nt < BN / 8; ++nt) {
      const __nv_bfloat16* Lr = Ls + (nt * 8 + g) * LDS + k;
      mma_bf16_16816(acc[nt], a0, a1, a2, a3, *reinterpret_cast<const uint32_t*>(Lr),
                     *reinterpret_cast<const uint32_t*>(Lr + 8));
    }
  }
  __syncthreads();   // Ts/Ls no longer needed: reuse the space for the fp32 tile
#pragma unroll
  for (int nt = 0; nt < BN / 8; ++nt) {
    const int col = nt * 8 + 2 * t, row = warp * 16 + g;
    Ys[row * BN + col] = acc[nt][0];
    Ys[row * BN + col + 1] = acc[nt][1];
    Ys[(row + 8) * BN + col] = acc[nt][2];
    Ys[(row + 8) * BN + col + 1] = acc[nt][3];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < BM * BN / 8; i += 128) {
    const int r = i / (BN / 8), c = (i % (BN / 8)) * 8;
    if (m0 + r >= M) continue;
    uint4* yp = reinterpret_cast<uint4*>(Y + (size_t)(m0 + r) * N + n0 + c);
    const uint4 y = *yp;
    const uint32_t w[4] = {y.x, y.y, y.z, y.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float lo = bf16lo(w[q]) + Ys[r * BN + c + 2 * q];
      const float hi = bf16hi(w[q]) + Ys[r * BN + c + 2 * q + 1];
      const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
      o[q] = *reinterpret_cast<const uint32_t*>(&p);
    }
    *yp = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace svdq
