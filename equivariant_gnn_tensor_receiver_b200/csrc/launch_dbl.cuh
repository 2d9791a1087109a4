// Launcher definitions of the double-backward edge streams (instantiated per RM in tu_*.cu).
#pragma once

#include <algorithm>

#include "launch_streams.cuh"
#include "streams_dbl.cuh"

namespace tpc {

template <int RM>
cudaError_t dbl_r_smem_rm(int bytes) {
  return cudaFuncSetAttribute(k_dbl_r_stream<RM>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int RM>
cudaError_t launch_dbl_r_rm(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                            const float* ggv, const float* x, const float* ggx, const float* G, const float* Gt,
                            float* dvec, cudaStream_t st) {
  const int threads = 32 * std::min(d.P, 16);
  k_dbl_r_stream<RM><<<unsigned(nc), threads, size_t(d.sm_floats2) * 4, st>>>(d, r0, nc, rowptr, col, vec, ggv,
                                                                              x, ggx, G, Gt, dvec);
  return cudaGetLastError();
}

}  // namespace tpc
