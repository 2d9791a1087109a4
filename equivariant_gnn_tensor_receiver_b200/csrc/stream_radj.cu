// Backward receiver adjoint stream (per-edge dY, db, dvec).
#include <algorithm>

#include "launchers.h"
#include "streams.cuh"

namespace tpc {

TPC_DEFINE_CG_UPLOADER(upload_cg_radj)

cudaError_t radj_set_smem_limit(int bytes) {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(k_radj_stream<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes))) return e;
  if ((e = cudaFuncSetAttribute(k_radj_stream<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes))) return e;
  return cudaFuncSetAttribute(k_radj_stream<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

cudaError_t launch_radj_stream(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col,
                               const float* vec, const float* x, const float* G, float* dvec, float* dY,
                               float* db, cudaStream_t st) {
  const int threads = 32 * std::min(d.P, 16);
  const size_t smem = size_t(d.sm_floats) * 4;
  if (d.rm == 4)
    k_radj_stream<4><<<unsigned(nc), threads, smem, st>>>(d, r0, nc, rowptr, col, vec, x, G, dvec, dY, db);
  else if (d.rm == 8)
    k_radj_stream<8><<<unsigned(nc), threads, smem, st>>>(d, r0, nc, rowptr, col, vec, x, G, dvec, dY, db);
  else
    k_radj_stream<16><<<unsigned(nc), threads, smem, st>>>(d, r0, nc, rowptr, col, vec, x, G, dvec, dY, db);
  return cudaGetLastError();
}

}  // namespace tpc
