// Launcher of the lane-per-edge adjoint stream (instantiated per RM in tu_adj_rm*.cu).
#pragma once

#include "launchers.h"
#include "streams_adj.cuh"

namespace tpc {

template <int RM>
cudaError_t adj_smem_rm(int bytes) {
  return cudaFuncSetAttribute(k_adj_stream<RM>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int RM>
cudaError_t launch_adj_rm(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                          const float* x, const float* G, float* dvec, float* dY, float* db, cudaStream_t st) {
  k_adj_stream<RM><<<unsigned(nc), 32 * d.fz_warps, d.adj_smem, st>>>(d, r0, nc, rowptr, col, vec, x, G, dvec, dY,
                                                                      db);
  return cudaGetLastError();
}

}  // namespace tpc
