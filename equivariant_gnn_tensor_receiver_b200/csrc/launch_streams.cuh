// Launcher definitions of the first-order edge streams (instantiated per RM in tu_*.cu).
#pragma once

#include <algorithm>

#include "launchers.h"
#include "streams.cuh"

namespace tpc {

template <int RM>
cudaError_t radj_smem_rm(int bytes) {
  return cudaFuncSetAttribute(k_radj_stream<RM>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int RM>
cudaError_t launch_radj_rm(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                           const float* x, const float* G, float* dvec, float* dY, float* db, cudaStream_t st) {
  const int threads = 32 * std::min(d.P, 16);
  k_radj_stream<RM><<<unsigned(nc), threads, size_t(d.sm_floats) * 4, st>>>(d, r0, nc, rowptr, col, vec, x, G,
                                                                            dvec, dY, db);
  return cudaGetLastError();
}

}  // namespace tpc

// Registers this unit's CG upload and shared-memory setter.
#define TPC_REGISTER_TU(tag, smem_fn)                                                              \
  namespace tpc {                                                                                  \
  static cudaError_t upload_##tag(const float* t) {                                                \
    return cudaMemcpyToSymbol(c_cg, t, sizeof(float) * kCgTotal);                                  \
  }                                                                                                \
  static TuRegistrar registrar_##tag(TuInit{&upload_##tag, smem_fn});                              \
  }
