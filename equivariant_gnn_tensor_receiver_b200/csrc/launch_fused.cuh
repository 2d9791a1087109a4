// Launchers of the fused forward / sender streams (instantiated per RM in tu_fused_*.cu).
#pragma once

#include "launch_streams.cuh"
#include "streams_v2.cuh"

namespace tpc {

template <int RM>
cudaError_t fwd_fused_smem_rm(int bytes) {
  cudaError_t e = cudaFuncSetAttribute(k_fwd_fused<RM, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e) return e;
  return cudaFuncSetAttribute(k_fwd_fused<RM, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int RM>
cudaError_t send_fused_smem_rm(int bytes) {
  cudaError_t e = cudaFuncSetAttribute(k_send_fused<RM, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e) return e;
  return cudaFuncSetAttribute(k_send_fused<RM, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int RM>
cudaError_t launch_fwd_rm(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                          const float* x, float* A, cudaStream_t st) {
  const int cw = 32 * d.fz_cpl_f;
  dim3 grid(unsigned(nc), unsigned((d.max_c_in + cw - 1) / cw));
  if (d.fz_cpl_f == 2)
    k_fwd_fused<RM, 2><<<grid, 32 * d.fz_warps, d.fz_smem_f, st>>>(d, r0, rowptr, col, vec, x, A);
  else
    k_fwd_fused<RM, 1><<<grid, 32 * d.fz_warps, d.fz_smem_f, st>>>(d, r0, rowptr, col, vec, x, A);
  return cudaGetLastError();
}

template <int RM>
cudaError_t launch_send_rm(const DevPlan& d, int s0, int nc, const int* s_rowptr, const int* perm,
                           const int* s_recv, const float* vec, const float* g, float* B, cudaStream_t st) {
  const int cw = 32 * d.fz_cpl_s;
  dim3 grid(unsigned(nc), unsigned((d.max_c_out + cw - 1) / cw));
  if (d.fz_cpl_s == 2)
    k_send_fused<RM, 2><<<grid, 32 * d.fz_warps, d.fz_smem_s, st>>>(d, s0, s_rowptr, perm, s_recv, vec, g, B);
  else
    k_send_fused<RM, 1><<<grid, 32 * d.fz_warps, d.fz_smem_s, st>>>(d, s0, s_rowptr, perm, s_recv, vec, g, B);
  return cudaGetLastError();
}

}  // namespace tpc
