// Launcher definitions of the double-backward edge streams (instantiated per RM in tu_*.cu).
#pragma once

#include <algorithm>

#include "launch_streams.cuh"
#include "streams_dbl.cuh"

namespace tpc {

template <int RM>
cudaError_t launch_dbl_a_rm(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                            const float* ggv, const float* x, const float* ggx, float* A1, float* A0,
                            cudaStream_t st) {
  for (int p = 0; p < d.P; ++p) {
    const DevPath& q = d.path[p];
    dim3 grid(unsigned((nc + kWarpsPerBlock - 1) / kWarpsPerBlock), unsigned((q.c_in + 31) / 32));
    switch (triple_id(q.l1, q.l2, q.l3)) {
#define TPC_CASE(a, b, c)                                                                                      \
  case triple_id(a, b, c):                                                                                     \
    k_dbl_a_path<a, b, c, RM><<<grid, 32 * kWarpsPerBlock, 0, st>>>(d, p, r0, nc, rowptr, col, vec, ggv, x, \
                                                                    ggx, A1, A0);                              \
    break;
      TPC_FOR_EACH_TRIPLE(TPC_CASE)
#undef TPC_CASE
      default: return cudaErrorInvalidValue;
    }
  }
  return cudaGetLastError();
}

template <int RM>
cudaError_t launch_dbl_s_rm(const DevPlan& d, int s0, int nc, const int* s_rowptr, const int* perm,
                            const int* s_recv, const float* vec, const float* ggv, const float* g, float* B1,
                            float* B0, cudaStream_t st) {
  for (int p = 0; p < d.P; ++p) {
    const DevPath& q = d.path[p];
    dim3 grid(unsigned((nc + kWarpsPerBlock - 1) / kWarpsPerBlock), unsigned((q.c_out + 31) / 32));
    switch (triple_id(q.l1, q.l2, q.l3)) {
#define TPC_CASE(a, b, c)                                                                                        \
  case triple_id(a, b, c):                                                                                       \
    k_dbl_s_path<a, b, c, RM><<<grid, 32 * kWarpsPerBlock, 0, st>>>(d, p, s0, nc, s_rowptr, perm, s_recv, vec, \
                                                                    ggv, g, B1, B0);                             \
    break;
      TPC_FOR_EACH_TRIPLE(TPC_CASE)
#undef TPC_CASE
      default: return cudaErrorInvalidValue;
    }
  }
  return cudaGetLastError();
}

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
