// Top-rank SVD split of the smoothed weight on the device (placeholder: the
// library currently requires caller-supplied factors).
#pragma once

#include <cuda_bf16.h>

#include "svdq.h"

namespace svdq {

inline size_t svd_workspace_bytes(int64_t, int64_t, int) { return 0; }

inline svdq_status svd_lowrank_factors(int64_t, int64_t, int, const __nv_bfloat16*, const float*, __nv_bfloat16*,
                                       __nv_bfloat16*, void*, cudaStream_t, void (*set_err)(const char*, ...)) {
  set_err("the device SVD is not built yet: pass SVDQ_PREPARE_GIVEN_FACTORS");
  return SVDQ_ERR_INVALID_ARG;
}

}  // namespace svdq
