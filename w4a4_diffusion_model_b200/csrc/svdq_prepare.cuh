// Offline weight preparation of the SVDQuant layer:
//   * smoothing_lambda_kernel: lambda_j = ax_j^alpha / aw_j^(1-alpha)
//     (anrans.github.io AI-infra handbook, Quantization chapter, SmoothQuant);
//   * residual_quantize_kernel: R = W_hat - (lambda L1') L2 in fp64, rounded to
//     fp32, then NVFP4-encoded along K (devpress.csdn.net SVDQuant
//     walkthrough, eq. (5)); the INT4 encoding of the same R is in
//     svdq_int4.cuh.
#pragma once

#include <cuda_bf16.h>

#include "svdq_quant.cuh"

namespace svdq {

// lambda64 = ax^alpha / aw^(1-alpha) (alpha = 0.5: sqrt on both sides, all
// steps correctly rounded), lambda = 1 where ax or aw is zero;
// lambda32 = fp32(lambda64), inv = fp32(1 / lambda32).
__global__ void smoothing_lambda_kernel(const float* __restrict__ act_amax, const float* __restrict__ w_amax,
                                        float alpha, float* __restrict__ lambda, float* __restrict__ inv_lambda,
                                        int K) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= K) return;
  const double ax = (double)act_amax[j], aw = (double)w_amax[j];
  double lam;
  if (ax == 0.0 || aw == 0.0) {
    lam = 1.0;
  } else if (alpha == 0.5f) {
    lam = __ddiv_rn(__dsqrt_rn(ax), __dsqrt_rn(aw));
  } else {
    lam = pow(ax, (double)alpha) / pow(aw, 1.0 - (double)alpha);
  }
  const float l32 = __double2float_rn(lam);
  lambda[j] = l32;
  inv_lambda[j] = __frcp_rn(l32);
}

// The fp32 residual of 16 consecutive input channels j0.. of output row n:
//   R[j][n] = fp32( lambda_j W[n][j] - sum_{k<r} (lambda_j L1p[k][j]) L2t[n][k] )
// with every product exact in fp64 and every addition rounded once, in
// increasing k.
__device__ __forceinline__ void residual_group16(const __nv_bfloat16* __restrict__ W, const float* __restrict__ lambda,
                                                 const __nv_bfloat16* __restrict__ L1p,
                                                 const __nv_bfloat16* __restrict__ L2t, int n, int j0, int K,
                                                 int rank, float (&v)[16]) {
  double lam[16], acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    lam[i] = (double)lambda[j0 + i];
    acc[i] = 0.0;
  }
  for (int k = 0; k < rank; ++k) {
    const double l2 = (double)__bfloat162float(L2t[(size_t)n * rank + k]);
    const __nv_bfloat16* l1 = L1p + (size_t)k * K + j0;
#pragma unroll
    for (int i = 0; i < 16; ++i)
      acc[i] = __dadd_rn(acc[i], __dmul_rn(__dmul_rn(lam[i], (double)__bfloat162float(l1[i])), l2));
  }
  const __nv_bfloat16* w = W + (size_t)n * K + j0;
#pragma unroll
  for (int i = 0; i < 16; ++i)
    v[i] = __double2float_rn(__dsub_rn(__dmul_rn(lam[i], (double)__bfloat162float(w[i])), acc[i]));
}

// One thread per (output row n, 16-group g of K): the residual's NVFP4 codes
// and scale byte.
__global__ void residual_quantize_kernel(const __nv_bfloat16* __restrict__ W, const float* __restrict__ lambda,
                                         const __nv_bfloat16* __restrict__ L1p,
                                         const __nv_bfloat16* __restrict__ L2t, uint8_t* __restrict__ Qr,
                                         uint8_t* __restrict__ Sr, int N, int K, int rank) {
  const int G = K >> 4;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)N * G) return;
  const int n = (int)(idx / G), g = (int)(idx % G);
  const int j0 = g * 16;
  float v[16];
  residual_group16(W, lambda, L1p, L2t, n, j0, K, rank, v);
  uint2 codes;
  uint32_t sb;
  nvfp4_encode16(v, codes, sb);
  *reinterpret_cast<uint2*>(Qr + (size_t)n * (K >> 1) + (j0 >> 1)) = codes;
  Sr[native_scale_offset(n, g, K)] = (uint8_t)sb;
}

}  // namespace svdq
