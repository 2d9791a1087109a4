// Launchers of the path-major streams (instantiated per RM in tu_pf_*.cu / tu_pm_*.cu).
#pragma once

#include "launch_streams.cuh"
#include "launchers.h"
#include "streams_pm.cuh"
#include "streams_pmf.cuh"

namespace tpc {

template <int RM, bool RECV, bool DBL>
cudaError_t pf_smem_rm(int bytes) {
  return cudaFuncSetAttribute(k_pf_stream<RM, RECV, DBL>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}
template <int RM>
cudaError_t pm_adj_smem_rm(int bytes) {
  return cudaFuncSetAttribute(k_pm_adj<RM>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}
template <int RM>
cudaError_t pm_dadj_smem_rm(int bytes) {
  return cudaFuncSetAttribute(k_pm_dadj<RM>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int RM>
cudaError_t launch_fwd_rm(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                          const float* x, float* A, cudaStream_t st) {
  k_pf_stream<RM, true, false><<<unsigned(nc), 32 * kPmWarps, d.pf_smem_r, st>>>(d, r0, rowptr, col, nullptr, vec,
                                                                                nullptr, x, nullptr, A, nullptr);
  return cudaGetLastError();
}

template <int RM>
cudaError_t launch_send_rm(const DevPlan& d, int s0, int nc, const int* s_rowptr, const int* perm,
                           const int* s_recv, const float* vec, const float* g, float* B, cudaStream_t st) {
  k_pf_stream<RM, false, false><<<unsigned(nc), 32 * kPmWarps, d.pf_smem_s, st>>>(d, s0, s_rowptr, s_recv, perm, vec,
                                                                                 nullptr, g, nullptr, B, nullptr);
  return cudaGetLastError();
}

template <int RM>
cudaError_t launch_dbl_a_rm(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                            const float* ggv, const float* x, const float* ggx, float* A1, float* A0,
                            cudaStream_t st) {
  k_pf_stream<RM, true, true><<<unsigned(nc), 32 * kPmWarps, d.pf_smem_r2, st>>>(d, r0, rowptr, col, nullptr, vec,
                                                                                ggv, x, ggx, A1, A0);
  return cudaGetLastError();
}

template <int RM>
cudaError_t launch_dbl_s_rm(const DevPlan& d, int s0, int nc, const int* s_rowptr, const int* perm,
                            const int* s_recv, const float* vec, const float* ggv, const float* g, float* B1,
                            float* B0, cudaStream_t st) {
  k_pf_stream<RM, false, true><<<unsigned(nc), 32 * kPmWarps, d.pf_smem_s2, st>>>(d, s0, s_rowptr, s_recv, perm, vec,
                                                                                 ggv, g, nullptr, B1, B0);
  return cudaGetLastError();
}

template <int RM>
cudaError_t launch_adj_rm(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                          const float* x, const float* G, float* dvec, float* dY, float* db, cudaStream_t st) {
  k_pm_adj<RM><<<unsigned(nc), 32 * kPmWarps, d.pm_smem_a, st>>>(d, r0, nc, rowptr, col, vec, x, G, dvec, dY, db);
  return cudaGetLastError();
}

template <int RM>
cudaError_t launch_dadj_rm(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                           const float* ggv, const float* x, const float* ggx, const float* G, const float* Gt,
                           float* dvec, cudaStream_t st) {
  k_pm_dadj<RM><<<unsigned(nc), 32 * kPmWarps, d.pm_smem_d, st>>>(d, r0, nc, rowptr, col, vec, ggv, x, ggx, G, Gt,
                                                                  dvec);
  return cudaGetLastError();
}

}  // namespace tpc
