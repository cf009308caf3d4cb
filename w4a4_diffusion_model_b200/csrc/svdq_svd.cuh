// Top-rank split of the smoothed weight on the device (devpress.csdn.net
// SVDQuant walkthrough, eq. (3)-(4): W_hat = L1 L2 + R with L1 L2 the best
// rank-r approximation, singular values folded into L1).
//
// W_hat = diag(lambda) W_lin^T is K x N and never formed: every product reads
// W_lin [N][K] bf16 and lambda directly. The top-r subspace comes from
// randomized subspace iteration (Halko, Martinsson and Tropp, "Finding
// structure with randomness", SIAM Review 2011, Algorithms 4.3/4.4 and 5.1):
//   Z = Omega (N x l Gaussian, l = r + oversampling)
//   Y = orth(W_hat Z); repeat q times { Z = orth(W_hat^T Y); Y = orth(W_hat Z) }
//   Z = W_hat^T Y  (= B^T, B = Y^T W_hat is l x N)
//   Z^T Z = B B^T = U~ S^2 U~^T  (symmetric eigenproblem, l x l)
//   L1 = Y U~_r S_r,  L2^T = Z U~_r S_r^-1
// orth() is SVQB (Stathopoulos and Wu, "A block orthogonalization procedure
// with constant synchronization requirements", SISC 2002) applied twice:
// G = Y^T Y = V D V^T, Y <- Y V D^-1/2, dropping null directions. The small
// eigenproblems use parallel cyclic Jacobi with round-robin pair ordering
// (Brent and Luk, SISC 1985) in one CTA. All arithmetic is fp32 with fixed
// reduction orders, so the factors are deterministic for a given input.
// Stored factors: L1p[k][j] = bf16(L1[j][k] / lambda_j), L2t[n][k] = bf16(L2[k][n]).
#pragma once

#include <cuda_bf16.h>

#include "svdq.h"
#include "svdq_quant.cuh"

namespace svdq {

constexpr int kSvdOversample = 32;
constexpr int kSvdPowerIters = 12;
constexpr int kSvdMaxL = 160;              // r <= 128 plus oversampling, multiple of 16
constexpr int kSvdTile = 64;               // output rows per CTA of the skinny products
constexpr int kSvdChunk = 32;              // reduction rows staged per iteration
constexpr int kSvdTargetCtas = 296;        // two CTAs per SM on 148 SMs (fixed: sizes the workspace)
constexpr int kSvdMaxSplit = 16;
constexpr int kSvdMaxGramParts = 64;
constexpr uint64_t kSvdSeed = 0x9E3779B97F4A7C15ull;

// Width of the sampled subspace: r + oversampling, at most min(K, N) and kSvdMaxL.
__host__ __device__ inline int svd_width(int64_t K, int64_t N, int r) {
  int64_t l = ((int64_t)r + kSvdOversample + 15) / 16 * 16;
  const int64_t mn = (K < N ? K : N) / 16 * 16;
  if (l > mn) l = mn;
  if (l > kSvdMaxL) l = kSvdMaxL;
  return (int)l;
}

// Split of the reduction dimension of a skinny product with `rows_out` output rows.
inline int svd_split(int64_t rows_out, int64_t red) {
  const int64_t tiles = rows_out / kSvdTile;
  int64_t s = (kSvdTargetCtas + tiles - 1) / tiles;
  const int64_t cap = red / 128 < kSvdMaxSplit ? red / 128 : kSvdMaxSplit;
  if (s > cap) s = cap;
  return s < 1 ? 1 : (int)s;
}

inline int svd_gram_parts(int64_t rows) {
  int64_t p = rows / 256;
  if (p > kSvdMaxGramParts) p = kSvdMaxGramParts;
  return p < 1 ? 1 : (int)p;
}

// ---------------------------------------------------------------- random start
// SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
// generators", OOPSLA 2014): counter-based, one 64-bit word per index.
__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  x += 0x9E3779B97F4A7C15ull;
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  return x ^ (x >> 31);
}

// Omega[i] ~ N(0, 1) by the Box-Muller transform of two 24-bit uniforms in (0, 1).
__global__ void svd_gaussian_kernel(float* __restrict__ out, size_t n, uint64_t seed) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const uint64_t h = splitmix64(seed ^ splitmix64(i));
    const float u1 = ((float)(uint32_t)(h >> 40) + 0.5f) * (1.0f / 16777216.0f);
    const float u2 = ((float)(uint32_t)((h >> 16) & 0xFFFFFFu) + 0.5f) * (1.0f / 16777216.0f);
    out[i] = sqrtf(-2.0f * logf(u1)) * cospif(2.0f * u2);
  }
}

// ---------------------------------------------------------------- skinny products
// Partial products over one slice of the reduction index b:
//   TRANS = false: part[s][j][c] = sum_{n in slice s} W[n][j] In[n][c]         (out rows j < K)
//   TRANS = true:  part[s][n][c] = sum_{j in slice s} W[n][j] lambda_j In[j][c] (out rows n < N)
// CTA (tile, s): 64 output rows x l columns; thread (ta = tid / 16, tc = tid % 16)
// owns rows 4 ta + [0, 4) and columns tc + 16 i.
template <bool TRANS>
__global__ void __launch_bounds__(256) svd_skinny_kernel(const __nv_bfloat16* __restrict__ W,
                                                         const float* __restrict__ lam, const float* __restrict__ In,
                                                         float* __restrict__ part, int N, int K, int l, int split) {
  constexpr int NCMAX = kSvdMaxL / 16;
  __shared__ __align__(16) float Wt[kSvdChunk][kSvdTile];   // [b][a]
  __shared__ __align__(16) float Xs[kSvdChunk * kSvdMaxL];  // [b][c], row stride l
  const int tid = threadIdx.x, ta = tid >> 4, tc = tid & 15;
  const int nc = l >> 4;
  const int rows_out = TRANS ? N : K, red = TRANS ? K : N;
  const int a0 = blockIdx.x * kSvdTile;
  const int s = blockIdx.y;
  const int per = red / kSvdChunk / split * kSvdChunk;   // the last slice takes the remainder
  const int b_begin = s * per, b_end = s == split - 1 ? red : b_begin + per;

  float acc[4][NCMAX];
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int i = 0; i < NCMAX; ++i) acc[k][i] = 0.f;

  for (int b0 = b_begin; b0 < b_end; b0 += kSvdChunk) {
    // W tile -> Wt[b][a] in fp32: 256 chunks of 8 bf16
    {
      uint4 v;
      int bb, aa;
      if (!TRANS) {   // rows b of W, 64 contiguous columns a
        bb = tid >> 3;
        aa = (tid & 7) * 8;
        v = __ldg(reinterpret_cast<const uint4*>(W + (size_t)(b0 + bb) * K + a0 + aa));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          Wt[bb][aa + 2 * e] = bf16lo(w[e]);
          Wt[bb][aa + 2 * e + 1] = bf16hi(w[e]);
        }
      } else {        // rows a of W, 32 contiguous columns b
        aa = tid >> 2;
        bb = (tid & 3) * 8;
        v = __ldg(reinterpret_cast<const uint4*>(W + (size_t)(a0 + aa) * K + b0 + bb));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          Wt[bb + 2 * e][aa] = bf16lo(w[e]);
          Wt[bb + 2 * e + 1][aa] = bf16hi(w[e]);
        }
      }
    }
    // input rows b0.. (scaled by lambda_b for TRANS)
    for (int e = tid * 4; e < kSvdChunk * l; e += 256 * 4) {
      const int bb = e / l, c = e % l;
      float4 x = *reinterpret_cast<const float4*>(In + (size_t)(b0 + bb) * l + c);
      if (TRANS) {
        const float lb = lam[b0 + bb];
        x.x *= lb; x.y *= lb; x.z *= lb; x.w *= lb;
      }
      *reinterpret_cast<float4*>(Xs + e) = x;
    }
    __syncthreads();
#pragma unroll 4
    for (int bb = 0; bb < kSvdChunk; ++bb) {
      const float4 w4 = *reinterpret_cast<const float4*>(&Wt[bb][4 * ta]);
      const float* xr = Xs + bb * l + tc;
#pragma unroll
      for (int i = 0; i < NCMAX; ++i) {
        if (i < nc) {
          const float x = xr[16 * i];
          acc[0][i] = fmaf(w4.x, x, acc[0][i]);
          acc[1][i] = fmaf(w4.y, x, acc[1][i]);
          acc[2][i] = fmaf(w4.z, x, acc[2][i]);
          acc[3][i] = fmaf(w4.w, x, acc[3][i]);
        }
      }
    }
    __syncthreads();
  }
  float* out = part + (size_t)s * rows_out * l;
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int i = 0; i < NCMAX; ++i)
      if (i < nc) out[(size_t)(a0 + 4 * ta + k) * l + tc + 16 * i] = acc[k][i];
}

// out[a][c] = scale_a * sum_{s in order} part[s][a][c]; scale_a = lambda_a when `lam` is given.
__global__ void svd_reduce_kernel(const float* __restrict__ part, const float* __restrict__ lam,
                                  float* __restrict__ out, int rows, int l, int split) {
  const size_t n = (size_t)rows * l;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
    float v = 0.f;
    for (int s = 0; s < split; ++s) v += part[(size_t)s * n + e];
    out[e] = lam ? v * lam[e / l] : v;
  }
}

// ---------------------------------------------------------------- Gram matrix
// part[p][c1][c2] = sum over row slice p of Y[row][c1] Y[row][c2] (Y is rows x l).
// Thread (ty = tid / 16, tx = tid % 16) owns c1 = ty + 16 i, c2 = tx + 16 j; both
// triangles are computed with the same products in the same order, so the sum
// is exactly symmetric.
__global__ void __launch_bounds__(256) svd_gram_kernel(const float* __restrict__ Y, float* __restrict__ part,
                                                       int rows, int l, int parts) {
  constexpr int NCMAX = kSvdMaxL / 16;
  __shared__ __align__(16) float Ys[kSvdChunk * kSvdMaxL];
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int nc = l >> 4;
  const int p = blockIdx.x;
  const int per = rows / kSvdChunk / parts * kSvdChunk;
  const int r_begin = p * per, r_end = p == parts - 1 ? rows : r_begin + per;
  float acc[NCMAX][NCMAX];
#pragma unroll
  for (int i = 0; i < NCMAX; ++i)
#pragma unroll
    for (int j = 0; j < NCMAX; ++j) acc[i][j] = 0.f;
  for (int r0 = r_begin; r0 < r_end; r0 += kSvdChunk) {
    for (int e = tid * 4; e < kSvdChunk * l; e += 256 * 4)
      *reinterpret_cast<float4*>(Ys + e) = *reinterpret_cast<const float4*>(Y + (size_t)r0 * l + e);
    __syncthreads();
    for (int rr = 0; rr < kSvdChunk; ++rr) {
      const float* yr = Ys + rr * l;
#pragma unroll
      for (int i = 0; i < NCMAX; ++i) {
        if (i < nc) {
          const float y1 = yr[ty + 16 * i];
#pragma unroll
          for (int j = 0; j < NCMAX; ++j)
            if (j < nc) acc[i][j] = fmaf(y1, yr[tx + 16 * j], acc[i][j]);
        }
      }
    }
    __syncthreads();
  }
  float* out = part + (size_t)p * l * l;
#pragma unroll
  for (int i = 0; i < NCMAX; ++i)
#pragma unroll
    for (int j = 0; j < NCMAX; ++j)
      if (i < nc && j < nc) out[(ty + 16 * i) * l + tx + 16 * j] = acc[i][j];
}

// ---------------------------------------------------------------- symmetric eigenproblem
constexpr int kJacobiThreads = 1024;
constexpr int kJacobiMaxSweeps = 15;

__host__ __device__ constexpr size_t jacobi_smem_bytes(int l) {
  return (size_t)(2 * l * l + l + 64) * sizeof(float) + (size_t)l * sizeof(int);
}

// Member `i` of round `st` of the round-robin schedule on l players (player 0 fixed).
__device__ __forceinline__ int rr_player(int k, int st, int l) { return k == 0 ? 0 : 1 + (k - 1 + st) % (l - 1); }

// G (l x l, symmetric) = V diag(D) V^T with D in descending order; one CTA.
// Each round rotates l/2 disjoint pairs (p, q) by the Jacobi rotation that
// zeroes A[p][q]: rows first (A <- J^T A), then columns (A <- A J, V <- V J).
__global__ void __launch_bounds__(kJacobiThreads) svd_jacobi_kernel(const float* __restrict__ G,
                                                                    float* __restrict__ Vout,
                                                                    float* __restrict__ Dout, int l) {
  extern __shared__ __align__(16) float jsm[];
  float* A = jsm;
  float* V = A + l * l;
  float* cs = V + l * l;          // c in [0, l/2), s in [l/2, l)
  float* red = cs + l;            // 64 floats
  int* order = reinterpret_cast<int*>(red + 64);
  const int tid = threadIdx.x, h = l / 2;
  for (int e = tid; e < l * l; e += kJacobiThreads) {
    A[e] = G[e];
    V[e] = (e / l == e % l) ? 1.f : 0.f;
  }
  __syncthreads();
  for (int sweep = 0; sweep < kJacobiMaxSweeps; ++sweep) {
    float off = 0.f, dia = 0.f;
    for (int e = tid; e < l * l; e += kJacobiThreads) {
      const int r = e / l, c = e % l;
      const float a = A[e];
      if (r < c) off = fmaf(a, a, off);
      else if (r == c) dia = fmaf(a, a, dia);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      off += __shfl_xor_sync(0xFFFFFFFFu, off, o);
      dia += __shfl_xor_sync(0xFFFFFFFFu, dia, o);
    }
    if ((tid & 31) == 0) {
      red[tid >> 5] = off;
      red[32 + (tid >> 5)] = dia;
    }
    __syncthreads();
    float off_t = 0.f, dia_t = 0.f;
    for (int w = 0; w < kJacobiThreads / 32; ++w) {
      off_t += red[w];
      dia_t += red[32 + w];
    }
    __syncthreads();
    if (off_t <= 1e-9f * dia_t) break;
    for (int st = 0; st < l - 1; ++st) {
      if (tid < h) {
        const int p = rr_player(tid, st, l), q = rr_player(l - 1 - tid, st, l);
        const float apq = A[p * l + q];
        float c = 1.f, s = 0.f;
        if (apq != 0.f) {
          const float th = (A[q * l + q] - A[p * l + p]) / (2.f * apq);
          const float t = copysignf(1.f, th) / (fabsf(th) + hypotf(th, 1.f));
          c = 1.f / sqrtf(fmaf(t, t, 1.f));
          s = t * c;
        }
        cs[tid] = c;
        cs[h + tid] = s;
      }
      __syncthreads();
      for (int e = tid; e < h * l; e += kJacobiThreads) {
        const int i = e / l, k = e % l;
        const int p = rr_player(i, st, l), q = rr_player(l - 1 - i, st, l);
        const float c = cs[i], s = cs[h + i];
        const float a = A[p * l + k], b = A[q * l + k];
        A[p * l + k] = c * a - s * b;
        A[q * l + k] = s * a + c * b;
      }
      __syncthreads();
      for (int e = tid; e < h * l; e += kJacobiThreads) {
        const int i = e / l, k = e % l;
        const int p = rr_player(i, st, l), q = rr_player(l - 1 - i, st, l);
        const float c = cs[i], s = cs[h + i];
        const float a = A[k * l + p], b = A[k * l + q];
        A[k * l + p] = c * a - s * b;
        A[k * l + q] = s * a + c * b;
        const float va = V[k * l + p], vb = V[k * l + q];
        V[k * l + p] = c * va - s * vb;
        V[k * l + q] = s * va + c * vb;
      }
      __syncthreads();
    }
  }
  if (tid < l) {   // descending order, ties by index
    const float d = A[tid * l + tid];
    int rank = 0;
    for (int j = 0; j < l; ++j) {
      const float dj = A[j * l + j];
      rank += (dj > d || (dj == d && j < tid)) ? 1 : 0;
    }
    order[rank] = tid;
  }
  __syncthreads();
  for (int e = tid; e < l * l; e += kJacobiThreads) Vout[e] = V[(e / l) * l + order[e % l]];
  if (tid < l) Dout[tid] = A[order[tid] * l + order[tid]];
}

// Small l x w transforms from (V, D):
//   factors == false (SVQB): T[c][k] = V[c][k] / sqrt(D[k]), or 0 for a null direction (w = l);
//   factors == true: T[c][k] = V[c][k] sigma_k and T2[c][k] = V[c][k] / sigma_k for k < w = r,
//   sigma_k = sqrt(D[k]); both 0 when sigma_k is negligible.
__global__ void svd_transform_kernel(const float* __restrict__ V, const float* __restrict__ D,
                                     float* __restrict__ T, float* __restrict__ T2, int l, int w, int factors) {
  const float d0 = D[0];
  for (int e = threadIdx.x; e < l * w; e += blockDim.x) {
    const int c = e / w, k = e % w;
    const float v = V[c * l + k], d = D[k];
    if (!factors) {
      T[e] = (d > 0.f && d > 1e-12f * d0) ? v / sqrtf(d) : 0.f;
    } else {
      const float sg = sqrtf(fmaxf(d, 0.f)), s0 = sqrtf(fmaxf(d0, 0.f));
      const bool keep = sg > 0.f && sg > 1e-6f * s0;
      T[e] = keep ? v * sg : 0.f;
      T2[e] = keep ? v / sg : 0.f;
    }
  }
}

// ---------------------------------------------------------------- Y T products
enum SvdApplyOut : int { kApplyF32 = 0, kApplyL1p = 1, kApplyL2t = 2 };

__host__ __device__ constexpr size_t apply_smem_bytes(int l, int w) {
  return (size_t)(l * w + l * kSvdTile) * sizeof(float);
}

// out = Y T with Y rows x l (fp32) and T l x w in shared memory. CTA: 64 rows;
// thread (ta, tc) owns rows 4 ta + [0, 4) and columns tc + 16 i. Output:
//   kApplyF32: out_f[row][k] (row stride w);
//   kApplyL1p: L1p[k][row] = bf16(value / lambda_row)   (rows = K);
//   kApplyL2t: L2t[row][k] = bf16(value)                 (rows = N).
template <int OUT>
__global__ void __launch_bounds__(256) svd_apply_kernel(const float* __restrict__ Y, const float* __restrict__ Tm,
                                                        const float* __restrict__ lam, float* __restrict__ out_f,
                                                        __nv_bfloat16* __restrict__ out_b, int rows, int l, int w) {
  constexpr int NCMAX = kSvdMaxL / 16;
  extern __shared__ __align__(16) float asmem[];
  float* Ts = asmem;               // [l][w]
  float* Ys = asmem + l * w;       // [l][64]: transposed row tile
  const int tid = threadIdx.x, ta = tid >> 4, tc = tid & 15;
  const int nw = w >> 4;
  const int a0 = blockIdx.x * kSvdTile;
  for (int e = tid; e < l * w; e += 256) Ts[e] = Tm[e];
  for (int e = tid; e < kSvdTile * l; e += 256) {
    const int rr = e / l, c = e % l;
    Ys[c * kSvdTile + rr] = Y[(size_t)(a0 + rr) * l + c];
  }
  __syncthreads();
  float acc[4][NCMAX];
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int i = 0; i < NCMAX; ++i) acc[k][i] = 0.f;
  for (int c = 0; c < l; ++c) {
    const float4 y4 = *reinterpret_cast<const float4*>(Ys + c * kSvdTile + 4 * ta);
    const float* tr = Ts + c * w + tc;
#pragma unroll
    for (int i = 0; i < NCMAX; ++i) {
      if (i < nw) {
        const float t = tr[16 * i];
        acc[0][i] = fmaf(y4.x, t, acc[0][i]);
        acc[1][i] = fmaf(y4.y, t, acc[1][i]);
        acc[2][i] = fmaf(y4.z, t, acc[2][i]);
        acc[3][i] = fmaf(y4.w, t, acc[3][i]);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int row = a0 + 4 * ta + k;
#pragma unroll
    for (int i = 0; i < NCMAX; ++i) {
      if (i >= nw) continue;
      const int col = tc + 16 * i;
      if (OUT == kApplyF32) out_f[(size_t)row * w + col] = acc[k][i];
      if (OUT == kApplyL1p) out_b[(size_t)col * rows + row] = __float2bfloat16_rn(__fdiv_rn(acc[k][i], lam[row]));
      if (OUT == kApplyL2t) out_b[(size_t)row * w + col] = __float2bfloat16_rn(acc[k][i]);
    }
  }
}

// ---------------------------------------------------------------- host driver
struct SvdPlan {
  int l, split_a, split_at, parts_y, parts_z;
  size_t off_ya, off_yb, off_za, off_zb, off_part, off_g, off_v, off_d, off_t, off_t2, bytes;
};

inline size_t svd_align(size_t x) { return (x + 255) / 256 * 256; }

inline SvdPlan svd_plan(int64_t K, int64_t N, int r) {
  SvdPlan p{};
  p.l = svd_width(K, N, r);
  p.split_a = svd_split(K, N);
  p.split_at = svd_split(N, K);
  p.parts_y = svd_gram_parts(K);
  p.parts_z = svd_gram_parts(N);
  const size_t l = (size_t)p.l, f = sizeof(float);
  size_t part = (size_t)p.split_a * K * l;
  if ((size_t)p.split_at * N * l > part) part = (size_t)p.split_at * N * l;
  if ((size_t)p.parts_y * l * l > part) part = (size_t)p.parts_y * l * l;
  if ((size_t)p.parts_z * l * l > part) part = (size_t)p.parts_z * l * l;
  size_t o = 0;
  p.off_ya = o; o += svd_align(K * l * f);
  p.off_yb = o; o += svd_align(K * l * f);
  p.off_za = o; o += svd_align(N * l * f);
  p.off_zb = o; o += svd_align(N * l * f);
  p.off_part = o; o += svd_align(part * f);
  p.off_g = o; o += svd_align(l * l * f);
  p.off_v = o; o += svd_align(l * l * f);
  p.off_d = o; o += svd_align(l * f);
  p.off_t = o; o += svd_align(l * l * f);
  p.off_t2 = o; o += svd_align(l * l * f);
  p.bytes = o;
  return p;
}

inline size_t svd_workspace_bytes(int64_t K, int64_t N, int r) { return r > 0 ? svd_plan(K, N, r).bytes : 0; }

}  // namespace svdq
