// C ABI of the SVDQuant W4A4 linear layer (declared in include/svdq.h):
// argument checks, tensor-map construction and kernel launches. The kernels
// live in the headers included below; this file is the library's single
// translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>

#include "svdq.h"
#include "svdq_deltaquant.cuh"
#include "svdq_gemm.cuh"
#include "svdq_gemm_pair.cuh"
#include "svdq_int4.cuh"
#include "svdq_prepare.cuh"
#include "svdq_quant.cuh"
#include "svdq_quant_tma.cuh"
#include "svdq_svd.cuh"

// Device scratch of svdq_prepare_weights_static: the SVD workspace for callers
// that provide none. Every byte a call reads is written earlier in that call.
static __device__ __align__(256) unsigned char g_prepare_scratch[SVDQ_STATIC_SCRATCH_BYTES];

namespace {

thread_local char g_last_error[512] = "";

svdq_status fail(svdq_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

#define SVDQ_CUDA(call)                                                                           \
  do {                                                                                            \
    cudaError_t e_ = (call);                                                                      \
    if (e_ != cudaSuccess) return fail(SVDQ_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_));   \
  } while (0)

#define SVDQ_LAUNCHED(what)                                                                       \
  do {                                                                                            \
    cudaError_t e_ = cudaGetLastError();                                                          \
    if (e_ != cudaSuccess) return fail(SVDQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e_));    \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

svdq_status check_shape(const svdq_shape& s) {
  if (s.M < 0 || s.K < 128 || s.N < 128 || s.K % 128 || s.N % 128 || s.rank < 0 || s.rank > 128 ||
      s.rank % 16)
    return fail(SVDQ_ERR_UNSUPPORTED_SHAPE,
                "shape M=%lld K=%lld N=%lld rank=%d: need M>=0, K,N multiples of 128, rank in {0,16,...,128}",
                (long long)s.M, (long long)s.K, (long long)s.N, (int)s.rank);
  if (s.M > (1ll << 31) - 1 || s.K > (1ll << 20) || s.N > (1ll << 24))
    return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "shape too large for 32-bit tile coordinates");
  return SVDQ_OK;
}

// Device check (compute capability 10.0), cached per device ordinal.
svdq_status check_device() {
  static std::mutex mu;
  static int cached[64];   // 0 unknown, 1 ok, 2 bad
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return fail(SVDQ_ERR_NO_DEVICE, "no CUDA device");
  }
  if (dev < 64) {
    std::lock_guard<std::mutex> lk(mu);
    if (cached[dev] == 0) {
      int major = 0, minor = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return fail(SVDQ_ERR_NO_DEVICE, "cannot query device %d", dev);
      }
      cached[dev] = (major == 10 && minor == 0) ? 1 : 2;
    }
    if (cached[dev] != 1) return fail(SVDQ_ERR_NO_DEVICE, "device %d is not compute capability 10.0 (sm_100a)", dev);
  }
  return SVDQ_OK;
}

// Per-device one-time state (kernel attributes, occupancy queries): a value
// per device ordinal, computed once under a lock by `init` with that device
// current and read lock-free afterwards. `init` returns a value > 0, or <= 0
// for a failure that is not cached (the next call retries).
constexpr int kMaxDevices = 64;

template <typename F>
int per_device_once(std::atomic<int> (&cache)[kMaxDevices], int dev, F init) {
  static std::mutex mu;
  if (dev < 0 || dev >= kMaxDevices) return init();
  const int v = cache[dev].load(std::memory_order_acquire);
  if (v > 0) return v;
  std::lock_guard<std::mutex> lk(mu);
  int w = cache[dev].load(std::memory_order_relaxed);
  if (w <= 0) {
    w = init();
    if (w > 0) cache[dev].store(w, std::memory_order_release);
  }
  return w;
}

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return dev;
}

// ---------------------------------------------------------------- tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// 2-D row-major tensor [rows][cols] of `elem_bytes`-sized elements, box of
// box_cols x box_rows, zero fill out of bounds.
svdq_status make_tmap(CUtensorMap* tm, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t cols,
                      uint64_t rows, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * (uint64_t)elem_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(tm, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return SVDQ_OK;
}

// Native scale buffer of `rows` (padded to 128) x K viewed as 3-D uint8
// [row blocks][K/64 * 2 chunks][256 bytes] (the atoms of one row block are
// contiguous, 512 bytes each); box of `blocks` row blocks x 8 chunks = 4 atoms.
svdq_status make_scale_tmap(CUtensorMap* tm, const void* base, int64_t rows, int64_t K, uint32_t blocks) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const uint64_t rb = (uint64_t)((rows + 127) / 128), chunks = (uint64_t)(K / 64) * 2;
  const cuuint64_t dims[3] = {256, chunks, rb};
  const cuuint64_t strides[2] = {256, chunks * 256};
  const cuuint32_t box[3] = {256, 8, blocks};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SVDQ_ERR_CUDA, "cuTensorMapEncodeTiled (scales) failed (%d)", (int)r);
  return SVDQ_OK;
}

size_t scale_bytes(int64_t rows, int64_t K) { return (size_t)((rows + 127) / 128) * (size_t)(K / 64) * 512u; }

// ---------------------------------------------------------------- launchers
int sm_count() {
  static std::atomic<int> cache[kMaxDevices];
  const int dev = current_device();
  const int n = per_device_once(cache, dev, [dev] {
    int v = 0;
    if (dev < 0 || cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    return v;
  });
  return n > 0 ? n : 148;
}

// Quantization: one CTA per BM rows (128 or 64) and K slice, one CTA per SM.
// Every configuration covers ceil(M/128)*128 rows, so the padding rows of the
// last scale atom get zero scales. With a low-rank branch the K slices of a
// row block form a cluster (their partial T is summed through distributed
// shared memory) and all clusters must be resident at once.
template <int RANK, int BM, int CODEC>
struct QuantLaunch {
  using L = svdq::QuantSmem<RANK, BM>;
  static constexpr auto kern = svdq::quantize_tma_kernel<RANK, BM, CODEC>;

  static svdq_status prepare() {   // once per device
    static std::atomic<int> done[kMaxDevices];
    cudaError_t err = cudaSuccess;
    per_device_once(done, current_device(), [&err] {
      err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
      return err == cudaSuccess ? 1 : 0;
    });
    if (err != cudaSuccess)
      return fail(SVDQ_ERR_CUDA, "cudaFuncSetAttribute(quantize_tma_kernel): %s", cudaGetErrorString(err));
    return SVDQ_OK;
  }

  // Clusters of k CTAs that can be resident at once, per device and k (cached
  // as count + 1, so that a device where none fit is cached too).
  static int max_clusters(int k) {
    static std::atomic<int> cache[3][kMaxDevices];
    const int i = k == 2 ? 0 : k == 4 ? 1 : 2;
    return per_device_once(cache[i], current_device(), [k] {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = k;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(k, 1, 1);
      cfg.blockDim = dim3(L::kThreads, 1, 1);
      cfg.dynamicSmemBytes = L::kBytes;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
      cudaGetLastError();
      return n + 1;
    }) - 1;
  }

  // Largest K split (8, 4, 2, 1) that keeps the grid in one wave; returns the
  // CTA count, 0 when K is not a whole number of stages.
  static int plan(const svdq_shape& s, int* ksplit) {
    *ksplit = 1;
    if (s.K % L::kCols) return 0;
    const int rowblocks = (int)((s.M + 127) / 128) * (128 / BM);
    const int nst = (int)(s.K / L::kCols);
    for (int k = 8; k >= 2; k /= 2) {
      if (nst % k || rowblocks * k > sm_count()) continue;
      if (RANK > 0 && rowblocks > max_clusters(k)) continue;
      *ksplit = k;
      return rowblocks * k;
    }
    *ksplit = 1;
    return rowblocks;
  }

  static svdq_status launch(const svdq_shape& s, int ksplit, const void* X, const float* inv, const void* L1p,
                            void* Qx, void* Sx, void* T, cudaStream_t st) {
    const int rowblocks = (int)((s.M + 127) / 128) * (128 / BM);
    CUtensorMap tx, tl;
    std::memset(&tl, 0, sizeof(tl));
    svdq_status r;
    if ((r = make_tmap(&tx, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)s.K, (uint64_t)s.M, 64, BM,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
      return r;
    if (RANK > 0 && (r = make_tmap(&tl, L1p, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)s.K, (uint64_t)RANK,
                                   64, RANK, CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
      return r;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = ksplit;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.gridDim = dim3(rowblocks * ksplit, 1, 1);
    cfg.blockDim = dim3(L::kThreads, 1, 1);
    cfg.dynamicSmemBytes = L::kBytes;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = (RANK > 0 && ksplit > 1) ? 2 : 1;
    SVDQ_CUDA(cudaLaunchKernelEx(&cfg, kern, tx, tl, inv, static_cast<uint8_t*>(Qx), static_cast<uint8_t*>(Sx),
                                 static_cast<__nv_bfloat16*>(T), (int)s.M, (int)s.K, ksplit));
    return SVDQ_OK;
  }
};

// 128-row CTAs unless 64-row CTAs put more of them in the one wave, or as
// many with a smaller K split (with a low-rank branch the slices of a row
// block form a cluster and add their partial T through distributed shared
// memory: fewer of them reduce faster; 1024 x 3072 rank 32: 7.53 -> 7.26 us).
template <int RANK, int CODEC>
svdq_status launch_quant_t(const svdq_shape& s, const void* X, const float* inv, const void* L1p, void* Qx, void* Sx,
                           void* T, cudaStream_t st) {
  using Big = QuantLaunch<RANK, 128, CODEC>;
  using Small = QuantLaunch<RANK, 64, CODEC>;
  if (s.M == 0) return SVDQ_OK;
  svdq_status r;
  if ((r = Big::prepare()) != SVDQ_OK || (r = Small::prepare()) != SVDQ_OK) return r;
  int kb = 1, ks = 1;
  const int nb = Big::plan(s, &kb), ns = Small::plan(s, &ks);
  if ((ns > nb || (RANK > 0 && ns == nb && ks < kb)) && ns <= sm_count())
    return Small::launch(s, ks, X, inv, L1p, Qx, Sx, T, st);
  return Big::launch(s, kb, X, inv, L1p, Qx, Sx, T, st);
}

template <int CODEC>
svdq_status launch_quant(const svdq_shape& s, int rank, const void* X, const float* inv, const void* L1p, void* Qx,
                         void* Sx, void* T, cudaStream_t st) {
  switch (rank) {
#define SVDQ_CASE(R) \
  case R:            \
    return launch_quant_t<R, CODEC>(s, X, inv, L1p, Qx, Sx, T, st);
    SVDQ_CASE(0) SVDQ_CASE(16) SVDQ_CASE(32) SVDQ_CASE(48) SVDQ_CASE(64) SVDQ_CASE(80) SVDQ_CASE(96)
    SVDQ_CASE(112) SVDQ_CASE(128)
#undef SVDQ_CASE
    default:
      return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "rank %d", rank);
  }
}

constexpr int kGemmStages = 3;

svdq_status launch_gemm_single(const svdq_shape& s, int rank, const void* Qx, const void* Sx, const void* T,
                               const void* Qr, const void* Sr, const void* L2t, void* Y, cudaStream_t st) {
  CUtensorMap tqx, tqr, tt, tl, ty;
  svdq_status r;
  if ((r = make_tmap(&tqx, Qx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)s.K / 2, (uint64_t)s.M, svdq::kGemmBKBytes,
                     svdq::kGemmBM, CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
    return r;
  if ((r = make_tmap(&tqr, Qr, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)s.K / 2, (uint64_t)s.N, svdq::kGemmBKBytes,
                     svdq::kGemmBN, CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
    return r;
  if (rank > 0) {
    if ((r = make_tmap(&tt, T, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)rank, (uint64_t)s.M, svdq::kGemmLrK,
                       svdq::kGemmBM, CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
      return r;
    if ((r = make_tmap(&tl, L2t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)rank, (uint64_t)s.N, svdq::kGemmLrK,
                       svdq::kGemmBN, CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
      return r;
  } else {
    memset(&tt, 0, sizeof(tt));
    memset(&tl, 0, sizeof(tl));
  }
  if ((r = make_tmap(&ty, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)s.N, (uint64_t)s.M, svdq::kEpiBoxCols, 32,
                     CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
    return r;
  using L = svdq::GemmSmem<kGemmStages>;
  auto kern = svdq::svdq_gemm_kernel<kGemmStages>;
  SVDQ_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes));
  const long long tiles = ((s.M + svdq::kGemmBM - 1) / svdq::kGemmBM) * ((s.N + svdq::kGemmBN - 1) / svdq::kGemmBN);
  const int grid = (int)(tiles < sm_count() ? tiles : sm_count());
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(svdq::kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = L::kBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  SVDQ_CUDA(cudaLaunchKernelEx(&cfg, kern, tqx, tqr, tt, tl, ty, static_cast<const uint8_t*>(Sx),
                               static_cast<const uint8_t*>(Sr), (int)s.M, (int)s.N, (int)s.K, rank));
  SVDQ_LAUNCHED("svdq_gemm_kernel");
  return SVDQ_OK;
}

// Launch configuration of the pair kernel: clusters of 2 CTAs, and (for real
// launches) programmatic stream serialization, so that the kernel's prologue
// overlaps the end of the previous kernel of the stream. `attr` must hold 2.
template <int NB, bool QLR = false>
cudaLaunchConfig_t pair_config(int clusters, cudaStream_t st, cudaLaunchAttribute* attr, bool pdl = true) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(svdq::kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = svdq::PairCfg<NB, QLR>::kBytes;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cfg;
}

// Clusters of the pair kernel (tile width NB) that fit on the device at once,
// cached per device; also sets the kernel's shared-memory attribute there.
template <int NB, bool QNEXT = false, bool QLR = false>
int pair_clusters() {
  static std::atomic<int> cache[kMaxDevices];
  // cached as count + 1; a failed attribute call is not cached
  return per_device_once(cache, current_device(), [] {
    auto kern = svdq::svdq_gemm_pair_kernel<NB, QNEXT, QLR>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, svdq::PairCfg<NB, QLR>::kBytes) !=
        cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = pair_config<NB, QLR>(sm_count() / 2, nullptr, attr, false);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, (void*)kern, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    return n + 1;
  }) - 1;
}

template <int NB, bool QNEXT = false, bool QLR = false>
svdq_status launch_gemm_pair(const svdq_shape& s, int rank, const void* Qx, const void* Sx, const void* T,
                             const void* Qr, const void* Sr, const void* L2t, void* Y, cudaStream_t st,
                             int clusters, const svdq::NextQuant& nq = svdq::NextQuant{}, bool store_y = true,
                             const void* next_L1p = nullptr) {
  constexpr uint32_t kBBox = NB == 256 ? 128 : 64;   // B rows per TMA box
  CUtensorMap tqx, tqr, tsa, tsb, tt, tl, ty, tl1n;
  memset(&tl1n, 0, sizeof(tl1n));
  svdq_status r;
  if ((r = make_tmap(&tqx, Qx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)s.K / 2, (uint64_t)s.M, svdq::kGemmBKBytes,
                     128, CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
    return r;
  if ((r = make_tmap(&tqr, Qr, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)s.K / 2, (uint64_t)s.N, svdq::kGemmBKBytes,
                     kBBox, CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
    return r;
  if ((r = make_scale_tmap(&tsa, Sx, s.M, s.K, 1)) != SVDQ_OK) return r;
  if ((r = make_scale_tmap(&tsb, Sr, s.N, s.K, NB / 128)) != SVDQ_OK) return r;
  if (rank > 0) {
    if ((r = make_tmap(&tt, T, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)rank, (uint64_t)s.M, svdq::kGemmLrK, 128,
                       CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
      return r;
    if ((r = make_tmap(&tl, L2t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)rank, (uint64_t)s.N, svdq::kGemmLrK,
                       kBBox, CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
      return r;
  } else {
    memset(&tt, 0, sizeof(tt));
    memset(&tl, 0, sizeof(tl));
  }
  if (store_y) {
    if ((r = make_tmap(&ty, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)s.N, (uint64_t)s.M, svdq::kEpiBoxCols,
                       32, CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
      return r;
  } else {
    memset(&ty, 0, sizeof(ty));
  }
  if (QLR) {   // the next layer's L1p' [next_rank][N]: boxes of 64 columns x next_rank/2 rows
    if ((r = make_tmap(&tl1n, next_L1p, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)s.N, (uint64_t)nq.next_rank,
                       64, (uint32_t)nq.next_rank / 2, CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
      return r;
  }
  auto kern = svdq::svdq_gemm_pair_kernel<NB, QNEXT, QLR>;
  const long long tiles = ((s.M + svdq::kPairBM - 1) / svdq::kPairBM) * (s.N / NB);
  const int ncl = (int)(tiles < clusters ? tiles : clusters);
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = pair_config<NB, QLR>(ncl, st, attr);
  SVDQ_CUDA(cudaLaunchKernelEx(&cfg, kern, tqx, tqr, tsa, tsb, tt, tl, ty, tl1n, (int)s.M, (int)s.N, (int)s.K, rank,
                               nq, store_y ? 1 : 0));
  SVDQ_LAUNCHED("svdq_gemm_pair_kernel");
  return SVDQ_OK;
}

// CTA pairs with 256 x 256 tiles when N is a multiple of 256, 256 x 384 tiles
// when it is a multiple of 384 only, otherwise the single-CTA kernel (also
// when pairs do not fit on the device). The 256-wide tiles keep a TMEM scale
// buffer per ring stage and measured as fast as or faster than the 384-wide
// ones on the FLUX projections. For small M the pair tiles leave most SMs
// idle; the single-CTA kernel's 128 x 256 tiles then occupy more of them, so
// it is chosen when it keeps at least 1.5x as many SMs busy.
// Which GEMM kernel serves shape s on the current device: 256 or 384 (CTA
// pairs with that tile width) or 128 (the single-CTA kernel).
int gemm_choice(const svdq_shape& s) {
  const long long sms = sm_count();
  const long long rows256 = (s.M + 255) / 256, rows128 = (s.M + 127) / 128;
  const int nb = s.N % 256 == 0 ? 256 : s.N % 384 == 0 ? 384 : 0;
  if (nb) {
    const long long pair_sms = 2 * rows256 * (s.N / nb), single_ctas = rows128 * ((s.N + 255) / 256);
    const long long busy_pair = pair_sms < sms ? pair_sms : sms, busy_single = single_ctas < sms ? single_ctas : sms;
    if (2 * busy_single >= 3 * busy_pair) return 128;
  }
  if (nb == 256 && pair_clusters<256>() > 0) return 256;
  if (s.N % 384 == 0 && pair_clusters<384>() > 0) return 384;
  return 128;
}

svdq_status launch_gemm(const svdq_shape& s, int rank, const void* Qx, const void* Sx, const void* T, const void* Qr,
                        const void* Sr, const void* L2t, void* Y, cudaStream_t st) {
  switch (gemm_choice(s)) {
    case 256: return launch_gemm_pair<256>(s, rank, Qx, Sx, T, Qr, Sr, L2t, Y, st, pair_clusters<256>());
    case 384: return launch_gemm_pair<384>(s, rank, Qx, Sx, T, Qr, Sr, L2t, Y, st, pair_clusters<384>());
    default: return launch_gemm_single(s, rank, Qx, Sx, T, Qr, Sr, L2t, Y, st);
  }
}

// The next layer's quantization runs in the GEMM epilogue when the shape takes
// the 256 x 256 pair kernel and the next layer's rank is 0, 16 or 32 (with a
// low-rank branch the epilogue also forms the partial T' of each tile, summed
// by tprime_reduce_kernel; svdq_gemm_qnext.cuh). Every other case forms Y (in
// the caller's Y or in the workspace) and runs the quantizer on it.
// The low-rank route is opt-in (SVDQ_NEXT_FUSE_LOWRANK): it measured slower
// than the two-call route on the FLUX projections.
bool qnext_fused(const svdq_shape& s, int next_rank, unsigned flags) {
  if (gemm_choice(s) != 256) return false;
  if (next_rank == 0) return pair_clusters<256, true>() > 0;
  return (flags & SVDQ_NEXT_FUSE_LOWRANK) && (next_rank == 16 || next_rank == 32) &&
         pair_clusters<256, true, true>() > 0;
}

size_t qnext_workspace_bytes(const svdq_shape& s, int next_rank, unsigned flags) {
  if (!qnext_fused(s, next_rank, flags)) return (size_t)s.M * (size_t)s.N * 2u;
  // fp32 partials of T' per 256-column tile: [N/256][M][next_rank]
  return (size_t)(s.N / 256) * (size_t)s.M * (size_t)next_rank * 4u;
}

template <int RANK>
svdq_status launch_up_rmw_t(const svdq_shape& s, const void* T, const void* L2t, void* Y, cudaStream_t st) {
  constexpr int LDS = RANK + 8;
  const size_t smem_in = (size_t)(64 + 128) * LDS * 2, smem_out = (size_t)64 * 128 * 4;
  const size_t smem = smem_in > smem_out ? smem_in : smem_out;
  auto kern = svdq::lowrank_up_rmw_kernel<RANK>;
  SVDQ_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  dim3 grid((unsigned)(s.N / 128), (unsigned)((s.M + 63) / 64));
  kern<<<grid, 128, smem, st>>>(static_cast<const __nv_bfloat16*>(T), static_cast<const __nv_bfloat16*>(L2t),
                                static_cast<__nv_bfloat16*>(Y), (int)s.M, (int)s.N);
  SVDQ_LAUNCHED("lowrank_up_rmw_kernel");
  return SVDQ_OK;
}

svdq_status launch_up_rmw(const svdq_shape& s, int rank, const void* T, const void* L2t, void* Y, cudaStream_t st) {
  switch (rank) {
#define SVDQ_CASE(R) \
  case R:            \
    return launch_up_rmw_t<R>(s, T, L2t, Y, st);
    SVDQ_CASE(16) SVDQ_CASE(32) SVDQ_CASE(48) SVDQ_CASE(64) SVDQ_CASE(80) SVDQ_CASE(96) SVDQ_CASE(112)
    SVDQ_CASE(128)
#undef SVDQ_CASE
    default:
      return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "rank %d", rank);
  }
}

// Randomized top-rank SVD of W_hat = diag(lambda) W_lin^T inside the caller's
// workspace (plan and kernels in svdq_svd.cuh); writes L1p [r][K] and L2t [N][r].
svdq_status launch_svd(const svdq_shape& s, const void* W, const float* lam, void* L1p, void* L2t, void* workspace,
                       cudaStream_t st) {
  using namespace svdq;
  const SvdPlan p = svd_plan(s.K, s.N, s.rank);
  const int K = (int)s.K, N = (int)s.N, l = p.l, r = s.rank;
  char* ws = static_cast<char*>(workspace);
  float* Y = reinterpret_cast<float*>(ws + p.off_ya);
  float* Yalt = reinterpret_cast<float*>(ws + p.off_yb);
  float* Z = reinterpret_cast<float*>(ws + p.off_za);
  float* Zalt = reinterpret_cast<float*>(ws + p.off_zb);
  float* part = reinterpret_cast<float*>(ws + p.off_part);
  float* G = reinterpret_cast<float*>(ws + p.off_g);
  float* V = reinterpret_cast<float*>(ws + p.off_v);
  float* D = reinterpret_cast<float*>(ws + p.off_d);
  float* T = reinterpret_cast<float*>(ws + p.off_t);
  float* T2 = reinterpret_cast<float*>(ws + p.off_t2);
  const __nv_bfloat16* Wb = static_cast<const __nv_bfloat16*>(W);
  {
    static std::atomic<int> done[kMaxDevices];
    cudaError_t err = cudaSuccess;
    per_device_once(done, current_device(), [&err] {
      const int big = (int)jacobi_smem_bytes(kSvdMaxL), ab = (int)apply_smem_bytes(kSvdMaxL, kSvdMaxL);
      if ((err = cudaFuncSetAttribute(svd_jacobi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, big)) ||
          (err = cudaFuncSetAttribute(svd_apply_kernel<kApplyF32>, cudaFuncAttributeMaxDynamicSharedMemorySize, ab)) ||
          (err = cudaFuncSetAttribute(svd_apply_kernel<kApplyL1p>, cudaFuncAttributeMaxDynamicSharedMemorySize, ab)) ||
          (err = cudaFuncSetAttribute(svd_apply_kernel<kApplyL2t>, cudaFuncAttributeMaxDynamicSharedMemorySize, ab)))
        return 0;
      return 1;
    });
    if (err != cudaSuccess) return fail(SVDQ_ERR_CUDA, "cudaFuncSetAttribute(svd kernels): %s", cudaGetErrorString(err));
  }
  auto grid_for = [](size_t n) { return (unsigned)((n + 255) / 256 < 2048 ? (n + 255) / 256 : 2048); };
  auto eig_of_gram = [&](const float* buf, int rows, int parts) -> svdq_status {
    svd_gram_kernel<<<parts, 256, 0, st>>>(buf, part, rows, l, parts);
    SVDQ_LAUNCHED("svd_gram_kernel");
    svd_reduce_kernel<<<grid_for((size_t)l * l), 256, 0, st>>>(part, nullptr, G, l, l, parts);
    SVDQ_LAUNCHED("svd_reduce_kernel");
    svd_jacobi_kernel<<<1, kJacobiThreads, jacobi_smem_bytes(l), st>>>(G, V, D, l);
    SVDQ_LAUNCHED("svd_jacobi_kernel");
    return SVDQ_OK;
  };
  auto svqb = [&](float*& buf, float*& alt, int rows, int parts) -> svdq_status {
    for (int pass = 0; pass < 2; ++pass) {
      svdq_status e = eig_of_gram(buf, rows, parts);
      if (e != SVDQ_OK) return e;
      svd_transform_kernel<<<1, 256, 0, st>>>(V, D, T, nullptr, l, l, 0);
      SVDQ_LAUNCHED("svd_transform_kernel");
      svd_apply_kernel<kApplyF32><<<rows / kSvdTile, 256, apply_smem_bytes(l, l), st>>>(buf, T, nullptr, alt,
                                                                                        nullptr, rows, l, l);
      SVDQ_LAUNCHED("svd_apply_kernel");
      float* t = buf;
      buf = alt;
      alt = t;
    }
    return SVDQ_OK;
  };
  auto prod = [&](bool trans, const float* in, float* out) -> svdq_status {
    const int rows = trans ? N : K, split = trans ? p.split_at : p.split_a;
    const dim3 grid(rows / kSvdTile, split);
    if (trans) svd_skinny_kernel<true><<<grid, 256, 0, st>>>(Wb, lam, in, part, N, K, l, split);
    else svd_skinny_kernel<false><<<grid, 256, 0, st>>>(Wb, lam, in, part, N, K, l, split);
    SVDQ_LAUNCHED("svd_skinny_kernel");
    svd_reduce_kernel<<<grid_for((size_t)rows * l), 256, 0, st>>>(part, trans ? nullptr : lam, out, rows, l, split);
    SVDQ_LAUNCHED("svd_reduce_kernel");
    return SVDQ_OK;
  };
  svdq_status e;
  svd_gaussian_kernel<<<grid_for((size_t)N * l), 256, 0, st>>>(Z, (size_t)N * l, kSvdSeed);
  SVDQ_LAUNCHED("svd_gaussian_kernel");
  if ((e = prod(false, Z, Y)) != SVDQ_OK || (e = svqb(Y, Yalt, K, p.parts_y)) != SVDQ_OK) return e;
  for (int it = 0; it < kSvdPowerIters; ++it) {
    if ((e = prod(true, Y, Z)) != SVDQ_OK || (e = svqb(Z, Zalt, N, p.parts_z)) != SVDQ_OK) return e;
    if ((e = prod(false, Z, Y)) != SVDQ_OK || (e = svqb(Y, Yalt, K, p.parts_y)) != SVDQ_OK) return e;
  }
  if ((e = prod(true, Y, Z)) != SVDQ_OK || (e = eig_of_gram(Z, N, p.parts_z)) != SVDQ_OK) return e;
  svd_transform_kernel<<<1, 256, 0, st>>>(V, D, T, T2, l, r, 1);
  SVDQ_LAUNCHED("svd_transform_kernel");
  svd_apply_kernel<kApplyL1p><<<K / kSvdTile, 256, apply_smem_bytes(l, r), st>>>(
      Y, T, lam, nullptr, static_cast<__nv_bfloat16*>(L1p), K, l, r);
  SVDQ_LAUNCHED("svd_apply_kernel");
  svd_apply_kernel<kApplyL2t><<<N / kSvdTile, 256, apply_smem_bytes(l, r), st>>>(
      Z, T2, nullptr, nullptr, static_cast<__nv_bfloat16*>(L2t), N, l, r);
  SVDQ_LAUNCHED("svd_apply_kernel");
  return SVDQ_OK;
}

svdq_status launch_channel_amax(int64_t rows, int64_t K, const void* X, float* amax, cudaStream_t st) {
  SVDQ_CUDA(cudaMemsetAsync(amax, 0, (size_t)K * sizeof(float), st));
  if (rows == 0) return SVDQ_OK;
  const int threads = 128;
  const int cols8 = (int)(K / 8);
  const int gx = (cols8 + threads - 1) / threads;
  // enough row blocks to fill the GPU several times over, each >= 32 rows
  int gy = (int)((rows + 31) / 32);
  const int max_gy = (4 * 148 + gx - 1) / gx;
  if (gy > max_gy) gy = max_gy;
  if (gy < 1) gy = 1;
  const int rows_per_block = (int)((rows + gy - 1) / gy);
  gy = (int)((rows + rows_per_block - 1) / rows_per_block);
  svdq::channel_amax_kernel<<<dim3(gx, gy), threads, 0, st>>>(static_cast<const __nv_bfloat16*>(X), amax, (int)rows,
                                                             (int)K, rows_per_block);
  SVDQ_LAUNCHED("channel_amax_kernel");
  return SVDQ_OK;
}

// ---------------------------------------------------------------- INT4 variant
size_t int4_act_scale_bytes(int64_t M, int64_t K) { return (size_t)(K / 64) * (size_t)((M + 127) / 128 * 128) * 4u; }

svdq_status launch_int4_gemm(const svdq_shape& s, const void* Qx, const void* Sx, const void* T, const void* Qr,
                             const void* Sr, const void* L2t, void* Y, cudaStream_t st) {
  CUtensorMap tqx, tqr, tt, tl;
  svdq_status r;
  if ((r = make_tmap(&tqx, Qx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)s.K, (uint64_t)s.M, svdq::kI4KTile,
                     svdq::kI4BM, CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
    return r;
  if ((r = make_tmap(&tqr, Qr, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)s.K, (uint64_t)s.N, svdq::kI4KTile,
                     svdq::kI4BN, CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
    return r;
  if (s.rank > 0) {
    if ((r = make_tmap(&tt, T, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)s.rank, (uint64_t)s.M, svdq::kGemmLrK,
                       svdq::kI4BM, CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
      return r;
    if ((r = make_tmap(&tl, L2t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)s.rank, (uint64_t)s.N,
                       svdq::kGemmLrK, svdq::kI4BN, CU_TENSOR_MAP_SWIZZLE_128B)) != SVDQ_OK)
      return r;
  } else {
    memset(&tt, 0, sizeof(tt));
    memset(&tl, 0, sizeof(tl));
  }
  auto kern = svdq::svdq_int4_gemm_kernel;
  SVDQ_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, svdq::kI4SmemBytes));
  const long long tiles = ((s.M + svdq::kI4BM - 1) / svdq::kI4BM) * ((s.N + svdq::kI4BN - 1) / svdq::kI4BN);
  const int grid = (int)(tiles < sm_count() ? tiles : sm_count());
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(svdq::kI4Threads, 1, 1);
  cfg.dynamicSmemBytes = svdq::kI4SmemBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  SVDQ_CUDA(cudaLaunchKernelEx(&cfg, kern, tqx, tqr, tt, tl, static_cast<const float*>(Sx),
                               static_cast<const float*>(Sr), static_cast<__nv_bfloat16*>(Y), (int)s.M, (int)s.N,
                               (int)s.K, (int)s.rank));
  SVDQ_LAUNCHED("svdq_int4_gemm_kernel");
  return SVDQ_OK;
}

}  // namespace

// ============================================================================ C ABI
extern "C" {

const char* svdq_status_string(int status) {
  switch (status) {
    case SVDQ_OK: return "SVDQ_OK";
    case SVDQ_ERR_INVALID_ARG: return "SVDQ_ERR_INVALID_ARG";
    case SVDQ_ERR_UNSUPPORTED_SHAPE: return "SVDQ_ERR_UNSUPPORTED_SHAPE";
    case SVDQ_ERR_MISALIGNED: return "SVDQ_ERR_MISALIGNED";
    case SVDQ_ERR_BUFFER_TOO_SMALL: return "SVDQ_ERR_BUFFER_TOO_SMALL";
    case SVDQ_ERR_NO_DEVICE: return "SVDQ_ERR_NO_DEVICE";
    case SVDQ_ERR_CUDA: return "SVDQ_ERR_CUDA";
    case SVDQ_ERR_TIMEOUT: return "SVDQ_ERR_TIMEOUT";
    case SVDQ_ERR_INTERNAL: return "SVDQ_ERR_INTERNAL";
    default: return "SVDQ_ERR_UNKNOWN";
  }
}

const char* svdq_last_error(void) { return g_last_error; }

int svdq_version(void) { return 100; }

svdq_status svdq_act_sizes(svdq_shape s, size_t* qx, size_t* sx, size_t* t) {
  svdq_status r = check_shape(s);
  if (r != SVDQ_OK) return r;
  if (qx) *qx = (size_t)s.M * (size_t)(s.K / 2);
  if (sx) *sx = scale_bytes(s.M, s.K);
  if (t) *t = (size_t)s.M * (size_t)s.rank * 2u;
  return SVDQ_OK;
}

svdq_status svdq_weight_sizes(svdq_shape s, size_t* qr, size_t* sr, size_t* l1p, size_t* l2t, size_t* ws) {
  svdq_status r = check_shape(s);
  if (r != SVDQ_OK) return r;
  if (qr) *qr = (size_t)s.N * (size_t)(s.K / 2);
  if (sr) *sr = scale_bytes(s.N, s.K);
  if (l1p) *l1p = (size_t)s.rank * (size_t)s.K * 2u;
  if (l2t) *l2t = (size_t)s.N * (size_t)s.rank * 2u;
  if (ws) *ws = svdq::svd_workspace_bytes(s.K, s.N, s.rank);
  return SVDQ_OK;
}

svdq_status svdq_channel_amax(int64_t M, int64_t K, const void* X, float* amax, void* stream) {
  g_last_error[0] = 0;
  if (M < 1 || K < 8 || K % 8 || K > (1ll << 30)) return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "amax shape M=%lld K=%lld", (long long)M, (long long)K);
  if (!X || !amax) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(X) || !aligned16(amax)) return fail(SVDQ_ERR_MISALIGNED, "X and amax must be 16-byte aligned");
  svdq_status r = check_device();
  if (r != SVDQ_OK) return r;
  return launch_channel_amax(M, K, X, amax, static_cast<cudaStream_t>(stream));
}

svdq_status svdq_prepare_weights(svdq_shape s, const void* W, const float* act_amax, float alpha, unsigned int flags,
                                 void* L1p, void* L2t, void* Qr, void* Sr, float* lambda, float* inv_lambda,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  g_last_error[0] = 0;
  svdq_status r = check_shape(s);
  if (r != SVDQ_OK) return r;
  if (!(alpha >= 0.f && alpha <= 1.f)) return fail(SVDQ_ERR_INVALID_ARG, "alpha must be in [0, 1]");
  if (flags & ~(unsigned)SVDQ_PREPARE_GIVEN_FACTORS) return fail(SVDQ_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if (!W || !act_amax || !Qr || !Sr || !lambda || !inv_lambda || (s.rank > 0 && (!L1p || !L2t)))
    return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  const void* ptrs[] = {W, act_amax, Qr, Sr, lambda, inv_lambda, L1p, L2t, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SVDQ_ERR_MISALIGNED, "every pointer must be 16-byte aligned");
  const bool given = (flags & SVDQ_PREPARE_GIVEN_FACTORS) != 0;
  const size_t need = given ? 0 : svdq::svd_workspace_bytes(s.K, s.N, s.rank);
  if (workspace_bytes < need || (need > 0 && !workspace))
    return fail(SVDQ_ERR_BUFFER_TOO_SMALL, "workspace of %zu bytes needed", need);
  if ((r = check_device()) != SVDQ_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // weight channel maxima into the lambda buffer, then lambda / inv_lambda
  if ((r = launch_channel_amax(s.N, s.K, W, inv_lambda, st)) != SVDQ_OK) return r;
  svdq::smoothing_lambda_kernel<<<(unsigned)((s.K + 255) / 256), 256, 0, st>>>(act_amax, inv_lambda, alpha, lambda,
                                                                              inv_lambda, (int)s.K);
  SVDQ_LAUNCHED("smoothing_lambda_kernel");
  if (s.rank > 0 && !given) {
    if ((r = launch_svd(s, W, lambda, L1p, L2t, workspace, st)) != SVDQ_OK) return r;
  }
  const long long n_threads = s.N * (s.K / 16);
  svdq::residual_quantize_kernel<<<(unsigned)((n_threads + 127) / 128), 128, 0, st>>>(
      static_cast<const __nv_bfloat16*>(W), lambda, static_cast<const __nv_bfloat16*>(L1p),
      static_cast<const __nv_bfloat16*>(L2t), static_cast<uint8_t*>(Qr), static_cast<uint8_t*>(Sr), (int)s.N,
      (int)s.K, (int)s.rank);
  SVDQ_LAUNCHED("residual_quantize_kernel");
  return SVDQ_OK;
}

svdq_status svdq_prepare_weights_static(svdq_shape s, const void* W, const float* act_amax, float alpha,
                                        unsigned int flags, void* L1p, void* L2t, void* Qr, void* Sr, float* lambda,
                                        float* inv_lambda, void* stream) {
  g_last_error[0] = 0;
  svdq_status r = check_shape(s);
  if (r != SVDQ_OK) return r;
  if (flags & ~(unsigned)SVDQ_PREPARE_GIVEN_FACTORS) return fail(SVDQ_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  const bool given = (flags & SVDQ_PREPARE_GIVEN_FACTORS) != 0;
  const size_t need = (given || s.rank == 0) ? 0 : svdq::svd_workspace_bytes(s.K, s.N, s.rank);
  if (need > SVDQ_STATIC_SCRATCH_BYTES)
    return fail(SVDQ_ERR_BUFFER_TOO_SMALL,
                "shape K=%lld N=%lld rank=%d needs %zu bytes of SVD scratch, the static scratch holds %zu: "
                "use svdq_prepare_weights with a caller workspace",
                (long long)s.K, (long long)s.N, (int)s.rank, need, (size_t)SVDQ_STATIC_SCRATCH_BYTES);
  void* scratch = nullptr;
  if (need > 0) {
    if ((r = check_device()) != SVDQ_OK) return r;
    // device address of the scratch, looked up once per device with that device current
    static std::mutex mu;
    static void* addr[64];
    int dev = 0;
    SVDQ_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return fail(SVDQ_ERR_INTERNAL, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev]) {
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_prepare_scratch);
      if (e != cudaSuccess || !p)
        return fail(SVDQ_ERR_CUDA, "cudaGetSymbolAddress(static scratch): %s", cudaGetErrorString(e));
      addr[dev] = p;
    }
    scratch = addr[dev];
  }
  return svdq_prepare_weights(s, W, act_amax, alpha, flags, L1p, L2t, Qr, Sr, lambda, inv_lambda, scratch, need,
                              stream);
}

svdq_status svdq_quantize_act(svdq_shape s, const void* X, const float* inv_lambda, const void* L1p, void* Qx,
                              void* Sx, void* T, int variant, void* stream) {
  g_last_error[0] = 0;
  svdq_status r = check_shape(s);
  if (r != SVDQ_OK) return r;
  if (variant != SVDQ_FUSED && variant != SVDQ_UNFUSED) return fail(SVDQ_ERR_INVALID_ARG, "variant %d", variant);
  if (s.M == 0) return SVDQ_OK;
  if (!X || !inv_lambda || !Qx || !Sx || (s.rank > 0 && (!L1p || !T))) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  const void* ptrs[] = {X, inv_lambda, Qx, Sx, L1p, T};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SVDQ_ERR_MISALIGNED, "every pointer must be 16-byte aligned");
  if ((r = check_device()) != SVDQ_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (variant == SVDQ_FUSED) return launch_quant<svdq::kCodecNvfp4>(s, s.rank, X, inv_lambda, L1p, Qx, Sx, T, st);
  if ((r = launch_quant<svdq::kCodecNvfp4>(s, 0, X, inv_lambda, nullptr, Qx, Sx, nullptr, st)) != SVDQ_OK) return r;
  if (s.rank == 0) return SVDQ_OK;
  return launch_quant<svdq::kCodecNone>(s, s.rank, X, nullptr, L1p, nullptr, nullptr, T, st);
}

svdq_status svdq_linear(svdq_shape s, const void* Qx, const void* Sx, const void* T, const void* Qr, const void* Sr,
                        const void* L2t, void* Y, int variant, void* stream) {
  g_last_error[0] = 0;
  svdq_status r = check_shape(s);
  if (r != SVDQ_OK) return r;
  if (variant != SVDQ_FUSED && variant != SVDQ_UNFUSED) return fail(SVDQ_ERR_INVALID_ARG, "variant %d", variant);
  if (s.M == 0) return SVDQ_OK;
  if (!Qx || !Sx || !Qr || !Sr || !Y || (s.rank > 0 && (!T || !L2t))) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  const void* ptrs[] = {Qx, Sx, T, Qr, Sr, L2t, Y};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SVDQ_ERR_MISALIGNED, "every pointer must be 16-byte aligned");
  if ((r = check_device()) != SVDQ_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (variant == SVDQ_FUSED) return launch_gemm(s, s.rank, Qx, Sx, T, Qr, Sr, L2t, Y, st);
  if ((r = launch_gemm(s, 0, Qx, Sx, nullptr, Qr, Sr, nullptr, Y, st)) != SVDQ_OK) return r;
  if (s.rank == 0) return SVDQ_OK;
  return launch_up_rmw(s, s.rank, T, L2t, Y, st);
}

svdq_status svdq_linear_quantize_next_workspace(svdq_shape s, int32_t next_rank, unsigned int flags, size_t* bytes) {
  g_last_error[0] = 0;
  svdq_status r = check_shape(s);
  if (r != SVDQ_OK) return r;
  if (flags & ~SVDQ_NEXT_FUSE_LOWRANK) return fail(SVDQ_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if (next_rank < 0 || next_rank > 128 || next_rank % 16)
    return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "next rank %d: need one of 0, 16, ..., 128", (int)next_rank);
  if (!bytes) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  if (s.M == 0) {
    *bytes = 0;
    return SVDQ_OK;
  }
  if ((r = check_device()) != SVDQ_OK) return r;
  *bytes = qnext_workspace_bytes(s, next_rank, flags);
  return SVDQ_OK;
}

svdq_status svdq_linear_quantize_next(svdq_shape s, const void* Qx, const void* Sx, const void* T, const void* Qr,
                                      const void* Sr, const void* L2t, int32_t next_rank,
                                      const float* next_inv_lambda, const void* next_L1p, void* next_Qx,
                                      void* next_Sx, void* next_T, void* Y, void* workspace, size_t workspace_bytes,
                                      unsigned int flags, void* stream) {
  g_last_error[0] = 0;
  svdq_status r = check_shape(s);
  if (r != SVDQ_OK) return r;
  if (flags & ~SVDQ_NEXT_FUSE_LOWRANK) return fail(SVDQ_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  const svdq_shape ns = {s.M, s.N, 128, next_rank};   // the next layer reads Y as its X (K' = N)
  if ((r = check_shape(ns)) != SVDQ_OK) return r;
  if (s.M == 0) return SVDQ_OK;
  if (!Qx || !Sx || !Qr || !Sr || (s.rank > 0 && (!T || !L2t)) || !next_inv_lambda || !next_Qx || !next_Sx ||
      (next_rank > 0 && (!next_L1p || !next_T)))
    return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  const void* ptrs[] = {Qx, Sx, T, Qr, Sr, L2t, next_inv_lambda, next_L1p, next_Qx, next_Sx, next_T, Y, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SVDQ_ERR_MISALIGNED, "every pointer must be 16-byte aligned");
  if ((r = check_device()) != SVDQ_OK) return r;
  const bool fused = qnext_fused(s, next_rank, flags);
  const size_t need = (Y && !fused) ? 0 : qnext_workspace_bytes(s, next_rank, flags);
  if (need > 0 && (workspace_bytes < need || !workspace))
    return fail(SVDQ_ERR_BUFFER_TOO_SMALL, "workspace of %zu bytes needed", need);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!fused) {   // Y (into the workspace unless the caller wants it), then the quantizer
    void* y = Y ? Y : workspace;
    if ((r = launch_gemm(s, s.rank, Qx, Sx, T, Qr, Sr, L2t, y, st)) != SVDQ_OK) return r;
    return launch_quant<svdq::kCodecNvfp4>(ns, next_rank, y, next_inv_lambda, next_L1p, next_Qx, next_Sx, next_T, st);
  }
  svdq::NextQuant nq;
  nq.inv_lambda = next_inv_lambda;
  nq.qx = static_cast<uint8_t*>(next_Qx);
  nq.sx = static_cast<uint8_t*>(next_Sx);
  nq.tp_ws = static_cast<float*>(workspace);
  nq.next_rank = next_rank;
  if (next_rank == 0)
    return launch_gemm_pair<256, true>(s, s.rank, Qx, Sx, T, Qr, Sr, L2t, Y, st, pair_clusters<256, true>(), nq,
                                       Y != nullptr);
  if ((r = launch_gemm_pair<256, true, true>(s, s.rank, Qx, Sx, T, Qr, Sr, L2t, Y, st, pair_clusters<256, true, true>(),
                                             nq, Y != nullptr, next_L1p)) != SVDQ_OK)
    return r;
  // T' = the tiles' partials added in tile order, rounded to bf16
  const long long n4 = s.M * (long long)next_rank / 4;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3((unsigned)((n4 + 255) / 256), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  SVDQ_CUDA(cudaLaunchKernelEx(&cfg, svdq::tprime_reduce_kernel, static_cast<const float4*>(workspace),
                               static_cast<__nv_bfloat16*>(next_T), n4, (int)(s.N / 256)));
  SVDQ_LAUNCHED("tprime_reduce_kernel");
  return SVDQ_OK;
}

namespace svdq {

// L2t_out[n][:r] = L2t[n], L2t_out[n][r:] = B[n]; 16-byte chunks (r, extra multiples of 16).
__global__ void append_l2t_kernel(const uint4* __restrict__ L2t, const uint4* __restrict__ B, uint4* __restrict__ out,
                                  int N, int r, int extra) {
  const int cr = r / 8, ce = extra / 8, co = cr + ce;   // 8 bf16 per chunk
  const size_t n_chunks = (size_t)N * co;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n_chunks; i += (size_t)gridDim.x * blockDim.x) {
    const size_t n = i / co;
    const int c = (int)(i % co);
    out[i] = c < cr ? L2t[n * cr + c] : B[n * ce + (c - cr)];
  }
}

// One thread waits on a barrier phase that never completes; the bounded wait
// gives up, records kDevErrSelfTest and the kernel returns.
__global__ void selftest_timeout_kernel() {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait(&bar, 0u, kDevErrSelfTest);   // gives up after kWaitLimitNs and records the code
  }
}

}  // namespace svdq

svdq_status svdq_append_lowrank(svdq_shape s, int32_t extra, const void* L1p, const void* L2t, const void* A,
                                const void* B, void* L1p_out, void* L2t_out, void* stream) {
  g_last_error[0] = 0;
  svdq_status r = check_shape(s);
  if (r != SVDQ_OK) return r;
  if (extra <= 0 || extra % 16 || s.rank + extra > 128)
    return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "rank %d + extra %d: need extra > 0, a multiple of 16, total <= 128",
                (int)s.rank, (int)extra);
  if (!A || !B || !L1p_out || !L2t_out || (s.rank > 0 && (!L1p || !L2t)))
    return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  const void* ptrs[] = {L1p, L2t, A, B, L1p_out, L2t_out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SVDQ_ERR_MISALIGNED, "every pointer must be 16-byte aligned");
  if ((r = check_device()) != SVDQ_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t l1_bytes = (size_t)s.rank * (size_t)s.K * 2u, a_bytes = (size_t)extra * (size_t)s.K * 2u;
  if (l1_bytes) SVDQ_CUDA(cudaMemcpyAsync(L1p_out, L1p, l1_bytes, cudaMemcpyDeviceToDevice, st));
  SVDQ_CUDA(cudaMemcpyAsync(static_cast<char*>(L1p_out) + l1_bytes, A, a_bytes, cudaMemcpyDeviceToDevice, st));
  const size_t chunks = (size_t)s.N * (size_t)((s.rank + extra) / 8);
  const unsigned grid = (unsigned)((chunks + 255) / 256 < 4096 ? (chunks + 255) / 256 : 4096);
  svdq::append_l2t_kernel<<<grid, 256, 0, st>>>(static_cast<const uint4*>(L2t), static_cast<const uint4*>(B),
                                                static_cast<uint4*>(L2t_out), (int)s.N, (int)s.rank, (int)extra);
  SVDQ_LAUNCHED("append_l2t_kernel");
  return SVDQ_OK;
}

svdq_status svdq_int4_act_sizes(svdq_shape s, size_t* qx, size_t* sx, size_t* t) {
  svdq_status r = check_shape(s);
  if (r != SVDQ_OK) return r;
  if (qx) *qx = (size_t)s.M * (size_t)s.K;
  if (sx) *sx = int4_act_scale_bytes(s.M, s.K);
  if (t) *t = (size_t)s.M * (size_t)s.rank * 2u;
  return SVDQ_OK;
}

svdq_status svdq_int4_weight_sizes(svdq_shape s, size_t* qr, size_t* sr) {
  svdq_status r = check_shape(s);
  if (r != SVDQ_OK) return r;
  if (qr) *qr = (size_t)s.N * (size_t)s.K;
  if (sr) *sr = (size_t)(s.K / 64) * (size_t)s.N * 4u;
  return SVDQ_OK;
}

svdq_status svdq_int4_quantize_residual(svdq_shape s, const void* W, const float* lambda, const void* L1p,
                                        const void* L2t, void* Qr, void* Sr, void* stream) {
  g_last_error[0] = 0;
  svdq_status r = check_shape(s);
  if (r != SVDQ_OK) return r;
  if (!W || !lambda || !Qr || !Sr || (s.rank > 0 && (!L1p || !L2t))) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  const void* ptrs[] = {W, lambda, L1p, L2t, Qr, Sr};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SVDQ_ERR_MISALIGNED, "every pointer must be 16-byte aligned");
  if ((r = check_device()) != SVDQ_OK) return r;
  const long long n_threads = s.N * (s.K / 16);
  svdq::residual_quantize_int4_kernel<<<(unsigned)((n_threads + 127) / 128), 128, 0,
                                        static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(W), lambda, static_cast<const __nv_bfloat16*>(L1p),
      static_cast<const __nv_bfloat16*>(L2t), static_cast<uint8_t*>(Qr), static_cast<float*>(Sr), (int)s.N, (int)s.K,
      (int)s.rank);
  SVDQ_LAUNCHED("residual_quantize_int4_kernel");
  return SVDQ_OK;
}

svdq_status svdq_int4_quantize_act(svdq_shape s, const void* X, const float* inv_lambda, const void* L1p, void* Qx,
                                   void* Sx, void* T, void* stream) {
  g_last_error[0] = 0;
  svdq_status r = check_shape(s);
  if (r != SVDQ_OK) return r;
  if (s.M == 0) return SVDQ_OK;
  if (!X || !inv_lambda || !Qx || !Sx || (s.rank > 0 && (!L1p || !T))) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  const void* ptrs[] = {X, inv_lambda, Qx, Sx, L1p, T};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SVDQ_ERR_MISALIGNED, "every pointer must be 16-byte aligned");
  if ((r = check_device()) != SVDQ_OK) return r;
  return launch_quant<svdq::kCodecInt4>(s, s.rank, X, inv_lambda, L1p, Qx, Sx, T, static_cast<cudaStream_t>(stream));
}

svdq_status svdq_int4_linear(svdq_shape s, const void* Qx, const void* Sx, const void* T, const void* Qr,
                             const void* Sr, const void* L2t, void* Y, void* stream) {
  g_last_error[0] = 0;
  svdq_status r = check_shape(s);
  if (r != SVDQ_OK) return r;
  if (s.M == 0) return SVDQ_OK;
  if (!Qx || !Sx || !Qr || !Sr || !Y || (s.rank > 0 && (!T || !L2t))) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  const void* ptrs[] = {Qx, Sx, T, Qr, Sr, L2t, Y};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SVDQ_ERR_MISALIGNED, "every pointer must be 16-byte aligned");
  if ((r = check_device()) != SVDQ_OK) return r;
  return launch_int4_gemm(s, Qx, Sx, T, Qr, Sr, L2t, Y, static_cast<cudaStream_t>(stream));
}

namespace {

svdq_status check_video_shape(int64_t F, int64_t H, int64_t W, int64_t C) {
  if (F < 1 || H < 1 || W < 1 || C < 64 || C % 64 || C > (1ll << 20) || F > (1ll << 31) || H > (1ll << 31) ||
      W > (1ll << 31) || F * H > (1ll << 31) || F * H * W > (1ll << 31) - 1)
    return fail(SVDQ_ERR_UNSUPPORTED_SHAPE,
                "video F=%lld H=%lld W=%lld C=%lld: need F, H, W >= 1, F*H*W < 2^31, C a multiple of 64 in [64, 2^20]",
                (long long)F, (long long)H, (long long)W, (long long)C);
  return SVDQ_OK;
}

int64_t video_blocks(int64_t F, int64_t H, int64_t W) { return ((F + 1) / 2) * ((H + 1) / 2) * ((W + 1) / 2); }

}  // namespace

svdq_status svdq_deltaquant_sizes(int64_t F, int64_t H, int64_t W, int64_t C, size_t* core_bytes, size_t* qd_bytes,
                                  size_t* sd_bytes) {
  g_last_error[0] = 0;
  svdq_status r = check_video_shape(F, H, W, C);
  if (r != SVDQ_OK) return r;
  const int64_t tokens = F * H * W;
  if (core_bytes) *core_bytes = (size_t)video_blocks(F, H, W) * (size_t)C;
  if (qd_bytes) *qd_bytes = (size_t)tokens * (size_t)(C / 2);
  if (sd_bytes) *sd_bytes = scale_bytes(tokens, C);
  return SVDQ_OK;
}

svdq_status svdq_deltaquant_encode(int64_t F, int64_t H, int64_t W, int64_t C, const void* X, void* core, void* Qd,
                                   void* Sd, void* stream) {
  g_last_error[0] = 0;
  svdq_status r = check_video_shape(F, H, W, C);
  if (r != SVDQ_OK) return r;
  if (!X || !core || !Qd || !Sd) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  const void* ptrs[] = {X, core, Qd, Sd};
  for (const void* p : ptrs)
    if (!aligned16(p)) return fail(SVDQ_ERR_MISALIGNED, "every pointer must be 16-byte aligned");
  if ((r = check_device()) != SVDQ_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t tokens = F * H * W;
  if (tokens % 128) {   // zero the last scale atom row block; the kernel writes its live rows
    const size_t atoms = (size_t)(C / 64) * 512u;
    SVDQ_CUDA(cudaMemsetAsync(static_cast<uint8_t*>(Sd) + (size_t)(tokens / 128) * atoms, 0, atoms, st));
  }
  const dim3 grid((unsigned)video_blocks(F, H, W),
                  (unsigned)((C / 16 + svdq::kDqGroupsPerCta - 1) / svdq::kDqGroupsPerCta));
  svdq::deltaquant_encode_kernel<<<grid, svdq::kDqThreads, 0, st>>>(
      static_cast<const __nv_bfloat16*>(X), static_cast<uint8_t*>(core), static_cast<uint8_t*>(Qd),
      static_cast<uint8_t*>(Sd), (int)F, (int)H, (int)W, (int)C);
  SVDQ_LAUNCHED("deltaquant_encode_kernel");
  return SVDQ_OK;
}

svdq_status svdq_selftest_timeout(void* stream) {
  g_last_error[0] = 0;
  svdq_status r = check_device();
  if (r != SVDQ_OK) return r;
  svdq::selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  SVDQ_LAUNCHED("selftest_timeout_kernel");
  return SVDQ_OK;
}

svdq_status svdq_scales_to_canonical(int64_t rows, int64_t K, const void* native, void* canonical, void* stream) {
  g_last_error[0] = 0;
  if (rows < 0 || K < 64 || K % 64 || K > (1ll << 20) || rows > (1ll << 31) - 1)
    return fail(SVDQ_ERR_UNSUPPORTED_SHAPE, "rows=%lld K=%lld", (long long)rows, (long long)K);
  if (rows == 0) return SVDQ_OK;
  if (!native || !canonical) return fail(SVDQ_ERR_INVALID_ARG, "null pointer");
  svdq_status r = check_device();
  if (r != SVDQ_OK) return r;
  const size_t n = (size_t)rows * (size_t)(K / 16);
  const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  svdq::scales_native_to_canonical_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(native), static_cast<uint8_t*>(canonical), (int)rows, (int)K);
  SVDQ_LAUNCHED("scales_native_to_canonical_kernel");
  return SVDQ_OK;
}

svdq_status svdq_check(void* stream) {
  g_last_error[0] = 0;
  svdq_status r = check_device();
  if (r != SVDQ_OK) return r;
  SVDQ_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  SVDQ_CUDA(cudaGetLastError());
  unsigned int word = 0, zero = 0;
  SVDQ_CUDA(cudaMemcpyFromSymbol(&word, svdq::g_device_error, sizeof(word)));
  if (word != 0) {
    SVDQ_CUDA(cudaMemcpyToSymbol(svdq::g_device_error, &zero, sizeof(zero)));
    return fail(SVDQ_ERR_TIMEOUT, "a kernel gave up on a bounded wait (device error %u)", word);
  }
  return SVDQ_OK;
}

}  // extern "C"
