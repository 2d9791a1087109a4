// Launcher of the lane-per-edge double-backward adjoint stream (per RM in tu_dadj_rm*.cu).
#pragma once

#include "launchers.h"
#include "streams_dadj.cuh"

namespace tpc {

template <int RM>
cudaError_t dadj_smem_rm(int bytes) {
  return cudaFuncSetAttribute(k_dadj_stream<RM>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int RM>
cudaError_t launch_dadj_rm(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                           const float* ggv, const float* x, const float* ggx, const float* G, const float* Gt,
                           float* dvec, cudaStream_t st) {
  k_dadj_stream<RM><<<unsigned(nc), 32 * d.fz_warps, d.dadj_smem, st>>>(d, r0, nc, rowptr, col, vec, ggv, x, ggx,
                                                                        G, Gt, dvec);
  return cudaGetLastError();
}

}  // namespace tpc
