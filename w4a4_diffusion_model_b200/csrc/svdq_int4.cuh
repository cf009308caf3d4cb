// The INT4 W4A4 variant of the SVDQuant layer (the pages' path for GPUs without
// NVFP4: devpress.csdn.net SVDQuant walkthrough, eq. (1) with q_max = 7 for
// signed 4-bit integers; anrans.github.io AI-infra handbook, Quantization
// chapter: one fp16 scale per 64 elements):
//   Y = bf16( sum_g  sx[m,g] sw[n,g] sum_{k in g} qx[m,k] qr[n,k]  +  T L2t^T )
//
// sm_100a has no 4-bit integer MMA and no block scaling with fp16 scales, so:
//   * the codes (integers in [-7, 7]) are held as E4M3 bytes, which represent
//     them exactly, and each 64-element group's integer products run as
//     tcgen05 kind::f8f6f4 MMAs (two of K = 32) into an fp32 TMEM buffer; the
//     sums are integers of magnitude <= 64 * 49, so they are exact;
//   * twelve rescale warps read each group's partial tile back and add it to
//     fp32 accumulators in registers with the group's scale pair:
//     acc += P * fp32(sx * sw) (the product of two fp16 values is exact in
//     fp32, so each group's term is rounded once, by the fused multiply-add);
//   * the low-rank up-projection T L2t^T runs as bf16 MMAs (kind::f16) into
//     one more partial buffer, added with weight 1.
// Two partial buffers alternate, so the MMAs of the next group run
// while the rescale warps drain the previous one. The rescale arithmetic
// (two fp32 operations per element and group) bounds the kernel, not the MMAs.
//
// Also here: the INT4 encoding of the weight residual.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "svdq_gemm_common.cuh"
#include "svdq_prepare.cuh"
#include "svdq_ptx.cuh"
#include "svdq_quant_tma.cuh"

namespace svdq {

// D(tmem) (+)= A(smem) * B(smem)^T with 8-bit float A/B, fp32 accumulate.
__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor, kind::f8f6f4 with E4M3 A/B (K-major), fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N) {
  return (1u << 4)                       // D format: f32
         | (0u << 7)                     // A format: E4M3
         | (0u << 10)                    // B format: E4M3
         | ((uint32_t)(N >> 3) << 17)    // N / 8
         | ((uint32_t)(M >> 4) << 24);   // M / 16
}

// d = a * b + c on fp32 pairs, each rounded once to nearest even.
__device__ __forceinline__ float2 fma2_rn(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ float2 add2_rn(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// 16 lanes x 256 bits, repeated 8 times along the columns: 32 registers per
// thread, laid out like mma.sync accumulators. For repetition j, thread t holds
//   r[4j], r[4j+1]:   lane base + t/4,     columns 8j + 2(t%4) + {0, 1}
//   r[4j+2], r[4j+3]: lane base + t/4 + 8, the same columns.
__device__ __forceinline__ void tmem_ld_16x256b_x8(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// tcgen05.wait::ld that the compiler sees as producing the loaded registers,
// so that no use of them is scheduled before the wait.
__device__ __forceinline__ void tmem_ld_wait_dep(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
        "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
        "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
        "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
}

// ---------------------------------------------------------------- weights
// One thread per (output row n, 16-element quarter of a 64-group of K); the
// four quarters of a group are the lanes of a quad. Codes: E4M3 bytes
// [N][K]; scales: fp32 [K/64][N]. Threads past the end work on the last quad's
// data (so that every quad shuffle has all its lanes) and store nothing.
__global__ void residual_quantize_int4_kernel(const __nv_bfloat16* __restrict__ W, const float* __restrict__ lambda,
                                              const __nv_bfloat16* __restrict__ L1p,
                                              const __nv_bfloat16* __restrict__ L2t, uint8_t* __restrict__ Qr,
                                              float* __restrict__ Sr, int N, int K, int rank) {
  const int G = K >> 4;
  const long long total = (long long)N * G;   // a multiple of 4 (K % 64 == 0)
  long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const bool live = idx < total;
  if (!live) idx = total - 4 + (threadIdx.x & 3);
  const int n = (int)(idx / G), g = (int)(idx % G);
  float v[16];
  residual_group16(W, lambda, L1p, L2t, n, 16 * g, K, rank, v);
  float2 v2[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v2[i] = make_float2(v[2 * i], v[2 * i + 1]);
  uint4 codes;
  float s;
  int4_encode_quarter(v2, codes, s);
  if (!live) return;
  *reinterpret_cast<uint4*>(Qr + (size_t)n * K + 16 * g) = codes;
  if ((g & 3) == 0) Sr[(size_t)(g >> 2) * N + n] = s;
}

// ---------------------------------------------------------------- GEMM
// Tiles of 128 x 192: twelve rescale warps of 64 columns (three per SM
// sub-partition) hide each other's TMEM-load latency within 128 registers.
constexpr int kI4BM = 128;
constexpr int kI4BN = 192;
constexpr int kI4KTile = 128;                        // K elements (= bytes) per k-tile: two groups
constexpr int kI4StageA = kI4BM * 128;               // 16 KB (also T: 128 x 64 bf16)
constexpr int kI4StageB = kI4BN * 128;               // 24 KB (also L2t: 192 x 64 bf16)
constexpr int kI4StageSx = 2 * kI4BM * 4;            // fp32 [2 groups][128 rows]
constexpr int kI4StageSw = 2 * kI4BN * 4;            // fp32 [2 groups][192 columns]
constexpr int kI4StageBytes = (kI4StageA + kI4StageB + kI4StageSx + kI4StageSw + 1023) / 1024 * 1024;   // 43 KB
constexpr int kI4Stages = 5;
constexpr int kI4RescaleWarps = 12;                  // warp w: lanes 32 (w % 4).., columns 64 (w / 4)..
constexpr int kI4Cols = kI4BN / (kI4RescaleWarps / 4);   // 64 accumulator columns per thread
constexpr int kI4ProducerWarp = 12;
constexpr int kI4MmaWarp = 13;
// 14 warps: at most 4 per SM sub-partition (16K registers each), so up to 128
// registers per thread
constexpr int kI4Threads = 32 * 14;
constexpr uint32_t kI4TmpStride = 256;               // TMEM columns between the two partial buffers
constexpr uint32_t kI4TmemCols = 512;
constexpr int kI4BarOffset = kI4Stages * kI4StageBytes;
constexpr int kI4SmemBytes = kI4BarOffset + 256 + 1024;   // barriers + alignment slack

// Persistent: one CTA per SM walks 128 x 256 output tiles (tile = blockIdx.x,
// blockIdx.x + gridDim.x, ...). Per tile, K/128 k-tiles of codes and scales,
// then ceil(r/64) low-rank k-tiles, through one ring. "Units" are what a
// partial buffer holds: each 64-element group, then the whole low-rank term.
// Barriers: full/empty per stage (empty: the MMA commit + every rescale warp,
// which read the stage's scales), tfull/tempty per partial buffer.
__global__ void __launch_bounds__(kI4Threads, 1) svdq_int4_gemm_kernel(
    const __grid_constant__ CUtensorMap tm_qx, const __grid_constant__ CUtensorMap tm_qr,
    const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_l2,
    const float* __restrict__ Sx, const float* __restrict__ Sw, __nv_bfloat16* __restrict__ Y, int M, int N, int K,
    int rank) {
  extern __shared__ __align__(1024) unsigned char i4_smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(i4_smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kI4BarOffset);
  uint64_t* empty = full + kI4Stages;
  uint64_t* tfull = empty + kI4Stages;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = (N + kI4BN - 1) / kI4BN;
  const int ntiles = ((M + kI4BM - 1) / kI4BM) * tiles_n;
  const int n_kt = K / kI4KTile;
  const int n_lr = (rank + kGemmLrK - 1) / kGemmLrK;
  const size_t ldsx = (size_t)((M + 127) & ~127);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kI4Stages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1 + kI4RescaleWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull + b, 1);
      mbar_init(tempty + b, kI4RescaleWarps);
    }
    mbar_init(mma_drain, 1);
    fence_mbar_init();
  }
  if (warp == kI4MmaWarp) {
    tmem_alloc(tmem_slot, kI4TmemCols);
    tmem_relinquish();
  }
  if (warp == kI4ProducerWarp && lane == 0) {
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

  if (warp == kI4ProducerWarp) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int m0 = (tile / tiles_n) * kI4BM, n0 = (tile % tiles_n) * kI4BN;
        const uint32_t sw_bytes = 4u * (uint32_t)min(kI4BN, N - n0);   // the last tile may be partial
        for (int kt = 0; kt < n_kt + n_lr; ++kt, ++it) {
          const int s = it % kI4Stages;
          if (!mbar_wait(empty + s, ((it / kI4Stages) & 1u) ^ 1u, kDevErrTimeoutEmpty)) {
            ok = false;
            break;
          }
          unsigned char* sa = smem + s * kI4StageBytes;
          unsigned char* sb = sa + kI4StageA;
          if (kt < n_kt) {
            unsigned char* ssx = sb + kI4StageB;
            unsigned char* ssw = ssx + kI4StageSx;
            mbar_arrive_expect_tx(full + s, (uint32_t)(kI4StageA + kI4StageB + kI4StageSx) + 2u * sw_bytes);
            tma_load_2d(sa, &tm_qx, full + s, kt * kI4KTile, m0);
            tma_load_2d(sb, &tm_qr, full + s, kt * kI4KTile, n0);
#pragma unroll
            for (int gi = 0; gi < 2; ++gi) {
              const size_t g = (size_t)(2 * kt + gi);
              bulk_load(ssx + gi * (kI4BM * 4), Sx + g * ldsx + m0, kI4BM * 4u, full + s);
              bulk_load(ssw + gi * (kI4BN * 4), Sw + g * (size_t)N + n0, sw_bytes, full + s);
            }
          } else {
            const int c = kt - n_kt;
            mbar_arrive_expect_tx(full + s, (uint32_t)(kI4StageA + kI4StageB));
            tma_load_2d(sa, &tm_t, full + s, c * kGemmLrK, m0);
            tma_load_2d(sb, &tm_l2, full + s, c * kGemmLrK, n0);
          }
        }
      }
      if (device_error_set()) {
        // Another role gave up: let the copies this thread issued land before
        // the CTA exits (bounded; only the last kI4Stages stages can be in flight).
        for (uint32_t j = it > (uint32_t)kI4Stages ? it - kI4Stages : 0u; j < it; ++j)
          mbar_drain(full + j % kI4Stages, (j / kI4Stages) & 1u);
      }
    }
  } else if (warp == kI4MmaWarp) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc = idesc_e4m3(kI4BM, kI4BN);
      constexpr uint32_t idesc_lr = idesc_bf16(kI4BM, kI4BN);
      uint32_t it = 0, u = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        for (int kt = 0; kt < n_kt && ok; ++kt, ++it) {
          const int s = it % kI4Stages;
          if (!mbar_wait(full + s, (it / kI4Stages) & 1u, kDevErrTimeoutFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * kI4StageBytes);
          const uint32_t sb = sa + kI4StageA;
#pragma unroll
          for (int gi = 0; gi < 2; ++gi, ++u) {
            const uint32_t b = u & 1u;
            if (!mbar_wait(tempty + b, ((u >> 1) & 1u) ^ 1u, kDevErrTimeoutAccum)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < 2; ++j) {   // 32 bytes (= 32 E4M3 elements) of K per MMA
              const uint64_t ad = smem_desc(sa + 64 * gi + 32 * j, 16, 1024, kSwizzle128B);
              const uint64_t bd = smem_desc(sb + 64 * gi + 32 * j, 16, 1024, kSwizzle128B);
              mma_f8(tmem + b * kI4TmpStride, ad, bd, idesc, (uint32_t)j);
            }
            tc_commit(tfull + b);
          }
          if (ok) tc_commit(empty + s);   // the stage's operands are free once these MMAs ran
        }
        if (!ok || n_lr == 0) continue;
        const uint32_t b = u & 1u;
        if (!mbar_wait(tempty + b, ((u >> 1) & 1u) ^ 1u, kDevErrTimeoutAccum)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int c = 0; c < n_lr; ++c, ++it) {
          const int s = it % kI4Stages;
          if (!mbar_wait(full + s, (it / kI4Stages) & 1u, kDevErrTimeoutFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * kI4StageBytes);
          const uint32_t sb = sa + kI4StageA;
          const int k16 = min(kGemmLrK, rank - c * kGemmLrK) / 16;
          for (int j = 0; j < k16; ++j) {
            const uint64_t ad = smem_desc(sa + 32 * j, 16, 1024, kSwizzle128B);
            const uint64_t bd = smem_desc(sb + 32 * j, 16, 1024, kSwizzle128B);
            mma_bf16(tmem + b * kI4TmpStride, ad, bd, idesc_lr, (c | j) != 0 ? 1u : 0u);
          }
          tc_commit(empty + s);
        }
        if (!ok) break;
        tc_commit(tfull + b);
        ++u;
      }
      if (!ok) {
        // Gave up: wait (bounded) for the MMAs already issued before TMEM is freed.
        tc_commit(mma_drain);
        mbar_drain(mma_drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------------ rescale warps
    // Warp w reads lane quarter q = w % 4 (rows 32q..32q+31 of the tile) and
    // column block cb = w / 4 (64 columns) with the 16x256b shape: thread t
    // owns rows 32q + 16h + t/4 + {0, 8} (h = 0, 1) and columns
    // 64cb + 8j + 2(t%4) + {0, 1} (j = 0..7), so it needs 16 weight scales and
    // 4 activation scales per group.
    const int q = warp & 3, cb = warp >> 2;
    const int tr = lane >> 2, tc = 2 * (lane & 3);
    const uint32_t quarter = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(kI4Cols * cb);
    float2 acc[2][8][2];   // [h][j][row +0 / +8]: a pair of adjacent columns
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[h][j][0] = acc[h][j][1] = make_float2(0.f, 0.f);
    uint32_t it = 0, u = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      const int m0 = (tile / tiles_n) * kI4BM, n0 = (tile % tiles_n) * kI4BN;
      for (int kt = 0; kt < n_kt && ok; ++kt, ++it) {
        const int s = it % kI4Stages;
        // the stage's scales have landed (the MMAs below imply it; this makes
        // the TMA writes visible to this warp)
        if (!mbar_wait(full + s, (it / kI4Stages) & 1u, kDevErrTimeoutFull)) {
          ok = false;
          break;
        }
        const float* ssx = reinterpret_cast<const float*>(smem + s * kI4StageBytes + kI4StageA + kI4StageB);
        const float* ssw = ssx + 2 * kI4BM;
#pragma unroll 1
        for (int gi = 0; gi < 2; ++gi, ++u) {
          const uint32_t b = u & 1u;
          if (!mbar_wait(tfull + b, (u >> 1) & 1u, kDevErrTimeoutAccum)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float* swp = ssw + gi * kI4BN + kI4Cols * cb + tc;
          const float* sxp = ssx + gi * kI4BM + 32 * q + tr;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t v[32];
            tmem_ld_16x256b_x8(quarter + ((uint32_t)(16 * h) << 16) + b * kI4TmpStride, v);
            tmem_ld_wait_dep(v);
            if (h == 1) {   // the partial buffer is read: the next unit's MMAs may overwrite it
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(tempty + b);
            }
            const float sx0 = sxp[16 * h], sx8 = sxp[16 * h + 8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float2 w2 = *reinterpret_cast<const float2*>(swp + 8 * j);
              const float2 c0 = mul2_rn(w2, make_float2(sx0, sx0));
              const float2 c8 = mul2_rn(w2, make_float2(sx8, sx8));
              acc[h][j][0] = fma2_rn(make_float2(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1])), c0,
                                     acc[h][j][0]);
              acc[h][j][1] = fma2_rn(make_float2(__uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3])),
                                     c8, acc[h][j][1]);
            }
          }
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + s);   // this warp no longer reads the stage's scales
      }
      if (!ok) break;
      if (n_lr > 0) {
        const uint32_t b = u & 1u;
        if (!mbar_wait(tfull + b, (u >> 1) & 1u, kDevErrTimeoutAccum)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t v[32];
          tmem_ld_16x256b_x8(quarter + ((uint32_t)(16 * h) << 16) + b * kI4TmpStride, v);
          tmem_ld_wait_dep(v);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            acc[h][j][0] = add2_rn(acc[h][j][0], make_float2(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1])));
            acc[h][j][1] =
                add2_rn(acc[h][j][1], make_float2(__uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3])));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(tempty + b);
          for (int c = 0; c < n_lr; ++c) mbar_arrive(empty + (it + c) % kI4Stages);
        }
        it += n_lr;
        ++u;
      }
      // Y: each (h, j, +0/+8) pair of adjacent columns is one 4-byte store
      const int col = n0 + kI4Cols * cb + tc;
      if (n0 + kI4Cols * cb < N) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int row = m0 + 32 * q + 16 * h + tr + 8 * r;
            if (row >= M) continue;
            __nv_bfloat16* dst = Y + (size_t)row * N + col;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<__nv_bfloat162*>(dst + 8 * j) = __floats2bfloat162_rn(acc[h][j][r].x, acc[h][j][r].y);
          }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[h][j][0] = acc[h][j][1] = make_float2(0.f, 0.f);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kI4MmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kI4TmemCols);
  }
}

}  // namespace svdq
