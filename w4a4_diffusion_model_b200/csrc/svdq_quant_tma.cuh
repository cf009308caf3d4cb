// Activation quantization with the fused low-rank down-projection, fed by a
// TMA ring (devpress.csdn.net SVDQuant walkthrough, eq. (1), eq. (5), Fig. 6:
// the down-projection shares the quantizer's read of X).
//
// A CTA owns BM (128 or 64) rows of X and a slice of K. One producer thread
// streams stages of 32 KB of X -- 16384/BM columns as 64-column x BM-row boxes
// with 128B swizzle -- with the matching columns of L1p (64-column boxes of
// RANK rows) and of inv_lambda, through a ring of stages (as many as fit in
// shared memory, at most six).
//
// Quantization: 16 warps own 16 rows and one 64-column slab of every stage
// each (with RG = BM/16 row groups, warp w takes rows 16 (w mod RG) + [0, 16)
// and slab w / RG). Thread (g = lane/4, t = lane%4) quantizes rows g and g+8,
// columns [16t, 16t+16) of the slab: one NVFP4 group per row, or a quarter of
// an INT4 group (64 elements; the four threads of a quad share it).
//
// Down-projection: one thread issues tcgen05 kind::f16 MMAs on the same
// shared-memory tiles (X box as A, L1p box as B, both K-major with 128B
// swizzle), accumulating T = X L1p^T over the CTA's K slice in TMEM
// (M = BM lanes, RANK fp32 columns). A stage is free once the quantizing warps
// have read it and the MMAs that read it have completed. Four warps read the
// accumulator back: with BM = 128 row r sits in TMEM lane r, with BM = 64 in
// lane (r mod 16) + 32 (r div 16).
//
// With K split over a cluster of `ksplit` CTAs the partial sums of T are added
// in cluster rank order through distributed shared memory: each CTA pushes its
// partial rows into the owning CTA's slots (or, for large ranks, peers read
// them remotely from the drained ring).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "svdq_ptx.cuh"
#include "svdq_quant.cuh"

namespace svdq {

constexpr int kQStageXBytes = 32768;       // X bytes per stage
constexpr int kQMaxStages = 6;
constexpr int kQSmemBudget = 227 * 1024 - 4096;   // leaves room for barriers, the 1 KB alignment and static tables

template <int RANK, int BM>
struct QuantSmem {
  static_assert(BM == 128 || BM == 64, "rows per CTA");
  static constexpr int kComputeWarps = 16;
  static constexpr int kProducerWarp = kComputeWarps;
  static constexpr int kMmaWarp = kComputeWarps + 1;
  static constexpr int kThreads = 32 * (kComputeWarps + 2);
  static constexpr int kRowGroups = BM / 16;
  static constexpr int kCols = kQStageXBytes / (2 * BM);       // K columns per stage
  static constexpr int kSlabs = kCols / 64;
  static_assert(kRowGroups * kSlabs == kComputeWarps, "one slab per warp and stage");
  static constexpr int kBoxBytes = 64 * BM * 2;
  static constexpr int kL1Box = 64 * RANK * 2;
  static constexpr int kL1 = kSlabs * kL1Box;
  static constexpr int kInv = kCols * 4;
  // 1 KB aligned stages: the 128B swizzle pattern repeats every 1024 bytes
  static constexpr int kStage = (kQStageXBytes + kL1 + kInv + 1023) / 1024 * 1024;
  static constexpr int kRedStride = RANK + 4;                  // fp32 partial T rows, padded against bank conflicts
  static constexpr int kRed = BM * kRedStride * 4;             // partial T of the K slices ([slice][row][col])
  // The partial sums get a region of their own (peers push into it while this
  // CTA may still be quantizing) when at least three stages still fit beside
  // it; otherwise they reuse the drained ring.
  static constexpr int kStagesSep = RANK > 0 ? (kQSmemBudget - kRed) / kStage : 0;
  static constexpr bool kRedSeparate = kStagesSep >= 3;
  static constexpr int kStagesMax = kRedSeparate ? kStagesSep : kQSmemBudget / kStage;
  static constexpr int kStages = kStagesMax < kQMaxStages ? kStagesMax : kQMaxStages;
  static constexpr int kRedOffset = kRedSeparate ? kStages * kStage : 0;
  static constexpr int kBarOffset = kStages * kStage + (kRedSeparate ? (kRed + 1023) / 1024 * 1024 : 0);
  static constexpr uint32_t kTmemCols = RANK <= 32 ? 32 : RANK <= 64 ? 64 : 128;
  static_assert(kRedSeparate || kRed <= kStages * kStage, "partial sums must fit in the ring");
  static_assert(kStages >= 2, "ring too shallow");
  static constexpr int kBytes = kBarOffset + 256 + 1024;
};

// TMA load of a 2-D box whose lines are marked first for eviction from L2:
// the quantizer reads each element of X exactly once, so X should not push
// the next kernel's operands out of L2.
__device__ __forceinline__ void tma_load_2d_once(void* dst, const void* tmap, uint64_t* bar, int x, int y) {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%3, %4}], [%2], %5;"
      ::"r"(smem_u32(dst)), "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(pol)
      : "memory");
}

// Byte offset of 16-byte chunk c of row r in a 128B-swizzled box (128-byte rows).
__device__ __forceinline__ uint32_t sw128(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// The NVFP4 recipe of nvfp4_encode16 for one group given as 8 packed bf16
// pairs and its 16 inverse smoothing factors (l[q] holds factors 4q..4q+3;
// smooth_group forms the products v):
//   v = fp32(x * inv_lambda); s = E4M3_rne_satfinite(fp32(max|v| / 6));
//   q = E2M1_rne_satfinite(v / s) of the exact quotient, all +0 when s is 0.
// The bracket (lo, hi) of 1/s comes from `rcp_tbl`, indexed by the E4M3 byte
// of s (recip_bracket of its value).
__device__ __forceinline__ void smooth_group(const uint32_t* w, const float4 (&l)[4], float2 (&v)[8]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    v[2 * q] = mul2_rn(make_float2(bf16lo(w[2 * q]), bf16hi(w[2 * q])), make_float2(l[q].x, l[q].y));
    v[2 * q + 1] = mul2_rn(make_float2(bf16lo(w[2 * q + 1]), bf16hi(w[2 * q + 1])), make_float2(l[q].z, l[q].w));
  }
}

__device__ __forceinline__ void encode_group_vals(const uint32_t* w, const float4 (&l)[4], const float2* rcp_tbl,
                                                  uint2& codes, uint32_t& sbyte) {
  float2 v[8];
  smooth_group(w, l, v);
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = fmaxf(fabsf(v[i].x), fabsf(v[i].y));
#pragma unroll
  for (int i = 0; i < 4; ++i) m[i] = fmaxf(m[i], m[i + 4]);
  m[0] = fmaxf(m[0], m[2]);
  m[1] = fmaxf(m[1], m[3]);
  const float amax = fmaxf(m[0], m[1]);
  const uint32_t b = (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(amax, 6.0f), __NV_SATFINITE, __NV_E4M3);
  sbyte = b;
  if (b == 0u) {
    codes = make_uint2(0u, 0u);
    return;
  }
  const float2 ib = rcp_tbl[b & 0x7Fu];
  uint32_t lo[2] = {0u, 0u}, hi[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    lo[i >> 2] |= (uint32_t)__nv_cvt_float2_to_fp4x2(mul2_rn(v[i], make_float2(ib.x, ib.x)), __NV_E2M1,
                                                     cudaRoundNearest) << (8 * (i & 3));
    hi[i >> 2] |= (uint32_t)__nv_cvt_float2_to_fp4x2(mul2_rn(v[i], make_float2(ib.y, ib.y)), __NV_E2M1,
                                                     cudaRoundNearest) << (8 * (i & 3));
  }
  if (((lo[0] ^ hi[0]) | (lo[1] ^ hi[1])) == 0u) {
    codes = make_uint2(lo[0], lo[1]);
    return;
  }
  const float sval = __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)b, __NV_E4M3)));
  codes = e2m1_group_exact(v, sval, make_uint2(lo[0], lo[1]), make_uint2(hi[0], hi[1]));
}

// The common path of encode_group_vals for one smoothed group v, without
// branches (so that the two groups of a thread interleave):
//   scale byte: amax times the bracket (lo, hi) of 1/6, both products
//   converted by one cvt; they give the same byte unless an E4M3 midpoint (or
//   the saturation bound) lies strictly between them, and then that byte is
//   the exact one (rounding is monotone);
//   codes: both bracket products of 1/s, from the table (e4m3_recip_bracket).
// `bad` is set when a pair disagrees; the caller then redoes the group with
// encode_group_vals (IEEE quotient for the scale, exact fix-up of the codes).
// A zero scale gives all +0 codes.
__device__ __forceinline__ void encode_group_fast(const float2 (&v)[8], float2 six, const float2* rcp_tbl,
                                                  uint2& codes, uint32_t& sbyte, uint32_t& bad) {
  const float m0 = max3_abs(v[0].x, v[0].y, v[1].x), m1 = max3_abs(v[1].y, v[2].x, v[2].y);
  const float m2 = max3_abs(v[3].x, v[3].y, v[4].x), m3 = max3_abs(v[4].y, v[5].x, v[5].y);
  const float m4 = max3_abs(v[6].x, v[6].y, v[7].x);
  const float amax = fmaxf(max3_abs(m0, m1, m2), max3_abs(m3, m4, v[7].y));
  const uint32_t two = (uint32_t)__nv_cvt_float2_to_fp8x2(mul2_rn(make_float2(amax, amax), six), __NV_SATFINITE,
                                                          __NV_E4M3);
  const uint32_t b = two & 0xFFu;
  const float2 ib = rcp_tbl[b & 0x7Fu];
  const uint32_t l0 = e2m1_word(v, ib.x), l1 = e2m1_word(v + 4, ib.x);
  const uint32_t h0 = e2m1_word(v, ib.y), h1 = e2m1_word(v + 4, ib.y);
  bad |= ((two >> 8) ^ b) | (l0 ^ h0) | (l1 ^ h1);
  codes = b != 0u ? make_uint2(l0, l1) : make_uint2(0u, 0u);
  sbyte = b;
}

// What the quantizing warps produce besides T.
enum QuantCodec : int {
  kCodecNone = 0,    // T only (the unfused variant's second pass)
  kCodecNvfp4 = 1,   // packed E2M1 codes, native E4M3 scale atoms
  kCodecInt4 = 2,    // INT4 codes as E4M3 bytes [M][K], fp32 scales [K/64][ceil(M/128)*128]
};

// The INT4 recipe (walkthrough eq. (1) with q_max = 7, one fp16 scale per 64
// elements) for 16 fp32 values a thread holds of a 64-element group; the
// group's four quarters sit in the four lanes of a quad (lane ^ 1, lane ^ 2):
//   s = fp16_rne(min(fp32(max|v| / 7), 65504)) (one rounding of the exact
//   quotient: an fp16 midpoint times 7 is exact in fp32);
//   q = clamp(RNE(v / s), -7, 7) of the exact quotient, all 0 when s is 0.
// The quotient is bracketed as for the E2M1 codes (recip_bracket); where the
// two products round to different integers k and k + 1 (in magnitude), |v| is
// compared with (k + 1/2) s, exact in fp32 (s has 11 significant bits).
// Codes are written as the E4M3 bytes of the integers (exact), the form the
// FP8 tensor-core MMA reads; the scale is returned as its fp32 value.
// Every lane of the warp must call it (quad shuffles).
__device__ __forceinline__ float int4_resolve(float v, float s, float qa, float qb) {
  const float m = fminf(fabsf(qa), fabsf(qb));
  const float t = __fmul_rn(m + 0.5f, s);   // exact
  const float x = fabsf(v);
  const float mag = x > t ? m + 1.f : x < t ? m : (fmodf(m, 2.f) == 0.f ? m : m + 1.f);
  return copysignf(mag, v);
}

__device__ __forceinline__ void int4_encode_quarter(const float2 (&v)[8], uint4& codes, float& scale) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fmaxf(fabsf(v[i].x), fabsf(v[i].y)));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
  const float s = __half2float(__float2half_rn(fminf(__fdiv_rn(amax, 7.0f), 65504.0f)));
  scale = s;
  if (s == 0.f) {
    codes = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const float2 ib = recip_bracket(s);
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 pl = mul2_rn(v[i], make_float2(ib.x, ib.x)), ph = mul2_rn(v[i], make_float2(ib.y, ib.y));
    float qx = rintf(pl.x), qy = rintf(pl.y);   // rint is half-to-even
    const float hx = rintf(ph.x), hy = rintf(ph.y);
    if (qx != hx) qx = int4_resolve(v[i].x, s, qx, hx);
    if (qy != hy) qy = int4_resolve(v[i].y, s, qy, hy);
    // adding +0 turns a -0 into +0 (code 0 is one byte, 0x00)
    const float2 qv = make_float2(__fadd_rn(fmaxf(fminf(qx, 7.f), -7.f), 0.f),
                                  __fadd_rn(fmaxf(fminf(qy, 7.f), -7.f), 0.f));
    b[i] = (uint32_t)__nv_cvt_float2_to_fp8x2(qv, __NV_SATFINITE, __NV_E4M3);
  }
  codes = make_uint4(b[0] | (b[1] << 16), b[2] | (b[3] << 16), b[4] | (b[5] << 16), b[6] | (b[7] << 16));
}

// The activation side: v = fp32(x * inv_lambda) for 8 packed bf16 pairs, then
// int4_encode_quarter.
__device__ __forceinline__ void encode_int4_quarter(const uint32_t* w, const float* il, uint4& codes, float& scale) {
  float2 v[8];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 l = *reinterpret_cast<const float4*>(il + 4 * q);
    v[2 * q] = mul2_rn(make_float2(bf16lo(w[2 * q]), bf16hi(w[2 * q])), make_float2(l.x, l.y));
    v[2 * q + 1] = mul2_rn(make_float2(bf16lo(w[2 * q + 1]), bf16hi(w[2 * q + 1])), make_float2(l.z, l.w));
  }
  int4_encode_quarter(v, codes, scale);
}

template <int RANK, int BM, int CODEC>
__global__ void __launch_bounds__(QuantSmem<RANK, BM>::kThreads, 1) quantize_tma_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_l1,
    const float* __restrict__ inv_lambda, uint8_t* __restrict__ Qx, uint8_t* __restrict__ Sx,
    __nv_bfloat16* __restrict__ T, int M, int K, int ksplit) {
  constexpr bool QUANT = CODEC != kCodecNone;
  if constexpr (!QUANT && RANK == 0) return;
  using L = QuantSmem<RANK, BM>;
  constexpr int RG = L::kRowGroups;
  extern __shared__ __align__(1024) unsigned char qsmem_raw[];
  __shared__ float2 rcp_tbl[128];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(qsmem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOffset);
  uint64_t* empty = full + L::kStages;
  uint64_t* acc_bar = empty + L::kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_bar + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kslice = blockIdx.x % ksplit;            // == cluster rank when ksplit > 1
  const int m0 = (blockIdx.x / ksplit) * BM;
  const int nst = K / L::kCols / ksplit;
  const int st0 = kslice * nst;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, (QUANT ? L::kComputeWarps : 0) + (RANK > 0 ? 1 : 0));
    }
    mbar_init(acc_bar, 1);
    fence_mbar_init();
  }
  if (CODEC == kCodecNvfp4 && threadIdx.x < 128) rcp_tbl[threadIdx.x] = e4m3_recip_bracket(threadIdx.x);
  if (RANK > 0 && warp == L::kMmaWarp) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  if (warp == L::kProducerWarp && lane == 0) {   // descriptors are kernel parameters: no dependency
    prefetch_tmap(&tm_x);
    if (RANK > 0) prefetch_tmap(&tm_l1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = RANK > 0 ? *tmem_slot : 0u;
  grid_dependency_wait();     // the previous kernel is complete (it may still read Qx, Sx, T or write X)
  grid_launch_dependents();

  if (warp == L::kProducerWarp) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      int j = 0;
      for (; j < nst; ++j) {
        const int s = j % L::kStages;
        if (!mbar_wait(empty + s, ((j / L::kStages) & 1u) ^ 1u, kDevErrTimeoutEmpty)) break;
        unsigned char* st = smem + s * L::kStage;
        const int c0 = (st0 + j) * L::kCols;
        mbar_arrive_expect_tx(full + s, (uint32_t)(kQStageXBytes + L::kL1 + (QUANT ? L::kInv : 0)));
#pragma unroll
        for (int b = 0; b < L::kSlabs; ++b) {
          tma_load_2d_once(st + b * L::kBoxBytes, &tm_x, full + s, c0 + 64 * b, m0);
          if (RANK > 0) tma_load_2d(st + kQStageXBytes + b * L::kL1Box, &tm_l1, full + s, c0 + 64 * b, 0);
        }
        if (QUANT) bulk_load(st + kQStageXBytes + L::kL1, inv_lambda + c0, (uint32_t)L::kInv, full + s);
      }
      if (device_error_set()) {   // let the copies issued land before the CTA exits
        for (int i = j > L::kStages ? j - L::kStages : 0; i < j; ++i)
          mbar_drain(full + i % L::kStages, (uint32_t)(i / L::kStages) & 1u);
      }
    }
  } else if (warp == L::kMmaWarp) {
    // ------------------------------------------------------------------ down-projection MMAs
    if (RANK > 0 && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(BM, RANK > 0 ? RANK : 16);
      bool ok = true;
      for (int j = 0; j < nst && ok; ++j) {
        const int s = j % L::kStages;
        if (!mbar_wait(full + s, (j / L::kStages) & 1u, kDevErrTimeoutFull)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = smem_u32(smem + s * L::kStage);
#pragma unroll
        for (int b = 0; b < L::kSlabs; ++b) {
          const uint32_t sa = st + b * L::kBoxBytes, sb = st + kQStageXBytes + b * L::kL1Box;
#pragma unroll
          for (int k = 0; k < 4; ++k) {   // 16 bf16 (32 bytes) of K per MMA
            const uint64_t ad = smem_desc(sa + 32 * k, 16, 1024, kSwizzle128B);
            const uint64_t bd = smem_desc(sb + 32 * k, 16, 1024, kSwizzle128B);
            mma_bf16(tmem, ad, bd, idesc, (j | b | k) != 0 ? 1u : 0u);
          }
        }
        tc_commit(empty + s);
      }
      tc_commit(acc_bar);
    }
  } else if (QUANT) {
    // ------------------------------------------------------------------ quantizing warps
    const int g = lane >> 2, t = lane & 3;
    const int rl = (warp % RG) * 16 + g;             // local rows rl and rl + 8
    const int h = warp / RG;                         // 64-column slab of every stage
    const int rA = m0 + rl, rB = rA + 8;
    const bool okA = rA < M, okB = rB < M;
    const size_t ldq = (size_t)K >> 1;
    const int cfirst = st0 * L::kCols + 64 * h + 16 * t;   // first column of this thread's group in stage 0
    uint8_t* qpa = Qx + (size_t)rA * ldq + (cfirst >> 1);
    uint8_t* qpb = Qx + (size_t)rB * ldq + (cfirst >> 1);
    uint8_t* spa = Sx + native_scale_offset(rA, cfirst >> 4, K);
    uint8_t* spb = Sx + native_scale_offset(rB, cfirst >> 4, K);
    const float2 six = recip_bracket(6.0f);
    for (int j = 0; j < nst; ++j) {
      const int s = j % L::kStages;
      if (!mbar_wait(full + s, (j / L::kStages) & 1u, kDevErrTimeoutFull)) break;
      const unsigned char* st = smem + s * L::kStage;
      const unsigned char* box = st + h * L::kBoxBytes;
      uint32_t xa[8], xb[8];
      {
        const uint4 a0 = *reinterpret_cast<const uint4*>(box + sw128(rl, 2 * t));
        const uint4 a1 = *reinterpret_cast<const uint4*>(box + sw128(rl, 2 * t + 1));
        const uint4 b0 = *reinterpret_cast<const uint4*>(box + sw128(rl + 8, 2 * t));
        const uint4 b1 = *reinterpret_cast<const uint4*>(box + sw128(rl + 8, 2 * t + 1));
        xa[0] = a0.x; xa[1] = a0.y; xa[2] = a0.z; xa[3] = a0.w;
        xa[4] = a1.x; xa[5] = a1.y; xa[6] = a1.z; xa[7] = a1.w;
        xb[0] = b0.x; xb[1] = b0.y; xb[2] = b0.z; xb[3] = b0.w;
        xb[4] = b1.x; xb[5] = b1.y; xb[6] = b1.z; xb[7] = b1.w;
      }
      const float* il = reinterpret_cast<const float*>(st + kQStageXBytes + L::kL1) + 64 * h + 16 * t;
      if constexpr (CODEC == kCodecInt4) {
        const int c = (st0 + j) * L::kCols + 64 * h + 16 * t;   // first column of this thread's group
        uint4 qa, qb;
        float sA, sB;
        encode_int4_quarter(xa, il, qa, sA);
        encode_int4_quarter(xb, il, qb, sB);
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + s);       // the stage's shared memory is no longer read
        if (okA) *reinterpret_cast<uint4*>(Qx + (size_t)rA * K + c) = qa;
        if (okB) *reinterpret_cast<uint4*>(Qx + (size_t)rB * K + c) = qb;
        if (t == 0) {   // rows past M (up to the 128-row padding) get zero scales: TMA zero-fills them
          float* S = reinterpret_cast<float*>(Sx) + (size_t)(c >> 6) * (size_t)((M + 127) & ~127);
          S[rA] = sA;
          S[rB] = sB;
        }
      } else {
        float4 l[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) l[q] = *reinterpret_cast<const float4*>(il + 4 * q);
        // The stage's shared memory has been read into registers: release it
        // before encoding (the arrive's release semantics order the loads
        // before it), so that its refill overlaps the work below.
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + s);
        float2 va[8], vb[8];
        smooth_group(xa, l, va);
        smooth_group(xb, l, vb);
        uint2 qa, qb;
        uint32_t sbA, sbB, bad = 0u;
        encode_group_fast(va, six, rcp_tbl, qa, sbA, bad);
        encode_group_fast(vb, six, rcp_tbl, qb, sbB, bad);
        if (bad != 0u) {   // a midpoint inside some bracket: the exact recipe for both groups
          encode_group_vals(xa, l, rcp_tbl, qa, sbA);
          encode_group_vals(xb, l, rcp_tbl, qb, sbB);
        }
        if (okA) *reinterpret_cast<uint2*>(qpa) = qa;
        if (okB) *reinterpret_cast<uint2*>(qpb) = qb;
        // rows past M get zero scales: TMA zero-fills them
        *spa = (uint8_t)sbA;
        *spb = (uint8_t)sbB;
        qpa += L::kCols / 2; qpb += L::kCols / 2;
        spa += (L::kCols / 64) * 512; spb += (L::kCols / 64) * 512;
      }
    }
  }

  if constexpr (RANK > 0) {
    // ------------------------------------------------------------------ T from TMEM
    // warp q < 4 reads TMEM lanes 32q..32q+31: rows 32q + lane (BM = 128) or
    // 16q + lane, lane < 16 (BM = 64) of this CTA's partial T
    const bool live = BM == 128 || lane < 16;
    const int r = BM == 128 ? 32 * warp + lane : 16 * warp + lane;
    const int rows_per = BM / ksplit;                // rows whose T this CTA finalises
    float* red = reinterpret_cast<float*>(smem + L::kRedOffset);
    if constexpr (L::kRedSeparate) {
      // Push: each CTA writes its partial rows straight into slot [kslice] of
      // the owning CTA's region (owner of row r: r / rows_per), so one cluster
      // barrier publishes everything and nothing is read remotely afterwards.
      if (warp < 4) {
        const bool acc_ok = mbar_wait(acc_bar, 0u, kDevErrTimeoutAccum);
        tc_fence_after();
        const int owner = r / rows_per, rr = r % rows_per;
        const uint32_t dst = mapa_shared(smem_u32(red + (kslice * rows_per + rr) * L::kRedStride), (uint32_t)owner);
#pragma unroll
        for (int c = 0; c < RANK / 16; ++c) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(tmem + ((uint32_t)(32 * warp) << 16) + 16u * c, v);
          tmem_ld_wait();
          if (!live || !acc_ok) continue;
          if (ksplit == 1) {
            if (m0 + r < M) {
              uint32_t p[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const __nv_bfloat162 bb =
                    __floats2bfloat162_rn(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                p[i] = *reinterpret_cast<const uint32_t*>(&bb);
              }
              uint4* out = reinterpret_cast<uint4*>(T + (size_t)(m0 + r) * RANK + 16 * c);
              out[0] = make_uint4(p[0], p[1], p[2], p[3]);
              out[1] = make_uint4(p[4], p[5], p[6], p[7]);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(dst + 64u * c + 16u * i),
                           "f"(__uint_as_float(v[4 * i])), "f"(__uint_as_float(v[4 * i + 1])),
                           "f"(__uint_as_float(v[4 * i + 2])), "f"(__uint_as_float(v[4 * i + 3]))
                           : "memory");
          }
        }
      }
      tc_fence_before();
      if (ksplit > 1) cluster_sync(); else __syncthreads();   // pushes visible; TMEM reads done
      if (warp == L::kMmaWarp) {
        mbar_drain(acc_bar, 0u);   // every down-projection MMA has completed (also after a failure)
        tc_fence_after();
        tmem_dealloc(tmem, L::kTmemCols);
      }
      if (ksplit > 1) {   // add the slices in rank order, from this CTA's own region
        const int cols4 = RANK / 4;
        for (int e = threadIdx.x; e < rows_per * cols4; e += L::kThreads) {
          const int row = e / cols4, c4 = (e % cols4) * 4;
          float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int p = 0; p < ksplit; ++p) {
            const float4 x = *reinterpret_cast<const float4*>(red + (p * rows_per + row) * L::kRedStride + c4);
            sum.x += x.x; sum.y += x.y; sum.z += x.z; sum.w += x.w;
          }
          const int grow = m0 + kslice * rows_per + row;
          if (grow < M) {
            const __nv_bfloat162 lo = __floats2bfloat162_rn(sum.x, sum.y), hi = __floats2bfloat162_rn(sum.z, sum.w);
            *reinterpret_cast<uint2*>(T + (size_t)grow * RANK + c4) =
                make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
          }
        }
      }
    } else {
      // Pull (large ranks): the partial rows reuse the drained ring; peers read
      // them remotely after a cluster barrier and keep them until a second one.
      __syncthreads();   // every role has left its loop: the ring is free once the MMAs are done
      if (warp < 4) {
        const bool acc_ok = mbar_wait(acc_bar, 0u, kDevErrTimeoutAccum);
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < RANK / 16; ++c) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(tmem + ((uint32_t)(32 * warp) << 16) + 16u * c, v);
          tmem_ld_wait();
          if (!live || !acc_ok) continue;
          if (ksplit == 1) {
            if (m0 + r < M) {
              uint32_t p[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const __nv_bfloat162 bb =
                    __floats2bfloat162_rn(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                p[i] = *reinterpret_cast<const uint32_t*>(&bb);
              }
              uint4* out = reinterpret_cast<uint4*>(T + (size_t)(m0 + r) * RANK + 16 * c);
              out[0] = make_uint4(p[0], p[1], p[2], p[3]);
              out[1] = make_uint4(p[4], p[5], p[6], p[7]);
            }
          } else {
            float4* dst = reinterpret_cast<float4*>(red + r * L::kRedStride + 16 * c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                   __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
          }
        }
      }
      tc_fence_before();
      __syncthreads();
      if (warp == L::kMmaWarp) {
        mbar_drain(acc_bar, 0u);   // every down-projection MMA has completed (also after a failure)
        tc_fence_after();
        tmem_dealloc(tmem, L::kTmemCols);
      }
      if (ksplit > 1) {
        cluster_sync();
        // CTA kslice finalises rows [kslice * BM / ksplit, ...), adding the slices in rank order
        const int e0 = kslice * rows_per * RANK, e1 = e0 + rows_per * RANK;
        const uint32_t red_addr = smem_u32(red);
        for (int e = e0 + (int)threadIdx.x; e < e1; e += L::kThreads) {
          const int row = e / RANK, col = e % RANK;
          const uint32_t off = 4u * (uint32_t)(row * L::kRedStride + col);
          float sum = 0.f;
          for (int p = 0; p < ksplit; ++p) {
            float x;
            const uint32_t a = mapa_shared(red_addr + off, (uint32_t)p);
            asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(x) : "r"(a) : "memory");
            sum += x;
          }
          if (m0 + row < M) T[(size_t)(m0 + row) * RANK + col] = __float2bfloat16_rn(sum);
        }
        cluster_sync();   // peers keep their partial sums until everyone has read them
      }
    }
  }
}

}  // namespace svdq
