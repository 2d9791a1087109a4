// Launchers of the warp-per-node edge streams (instantiated per (RM, LF[, CPL])
// in tu_wn_*.cu).  One warp per node of the chunk, kWnWarps nodes per CTA.
#pragma once

#include "launch_streams.cuh"
#include "launchers.h"
#include "streams_wn.cuh"
#include "streams_wna.cuh"

namespace tpc {

inline unsigned wn_grid(int nc) { return unsigned((nc + kWnWarps - 1) / kWnWarps); }
// path-major grid of the channel-lane streams
inline unsigned wn_grid_pm(const DevPlan& d, int nc) { return unsigned(d.P) * wn_grid(nc); }

template <int RM, int LF, int CPL, bool RECV, bool DBL>
cudaError_t wn_smem(int bytes) {
  cudaError_t e = cudaFuncSetAttribute(k_wn_stream<RM, LF, CPL, RECV, DBL, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if constexpr (DBL) {
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_wn_stream<RM, LF, CPL, RECV, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               bytes);
  }
  return e;
}
template <int RM, int LF, bool DBL>
cudaError_t wna_smem(int bytes) {
  cudaError_t e = cudaFuncSetAttribute(k_wn_adj<RM, LF, DBL, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       bytes);
  if constexpr (DBL) {
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_wn_adj<RM, LF, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  }
  return e;
}

template <int RM, int LF, int CPL>
cudaError_t launch_wn_fwd(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                          const float* x, float* A, cudaStream_t st) {
  if (nc <= 0) return cudaSuccess;
  k_wn_stream<RM, LF, CPL, true, false, false><<<wn_grid_pm(d, nc), 32 * kWnWarps, d.wn_smem_f, st>>>(
      d, r0, nc, rowptr, col, nullptr, vec, nullptr, x, nullptr, A, nullptr);
  return cudaGetLastError();
}

template <int RM, int LF, int CPL>
cudaError_t launch_wn_send(const DevPlan& d, int s0, int nc, const int* s_rowptr, const int* perm,
                           const int* s_recv, const float* vec, const float* g, float* B, cudaStream_t st) {
  if (nc <= 0) return cudaSuccess;
  k_wn_stream<RM, LF, CPL, false, false, false><<<wn_grid_pm(d, nc), 32 * kWnWarps, d.wn_smem_s, st>>>(
      d, s0, nc, s_rowptr, s_recv, perm, vec, nullptr, g, nullptr, B, nullptr);
  return cudaGetLastError();
}

template <int RM, int LF>
cudaError_t launch_wn_dbla(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                           const float* ggv, const float* x, const float* ggx, float* A1, float* A0,
                           cudaStream_t st) {
  if (nc <= 0) return cudaSuccess;
  if (A0)
    k_wn_stream<RM, LF, 1, true, true, true><<<wn_grid_pm(d, nc), 32 * kWnWarps, d.wn_smem_f2, st>>>(
        d, r0, nc, rowptr, col, nullptr, vec, ggv, x, ggx, A1, A0);
  else
    k_wn_stream<RM, LF, 1, true, true, false><<<wn_grid_pm(d, nc), 32 * kWnWarps, d.wn_smem_f2, st>>>(
        d, r0, nc, rowptr, col, nullptr, vec, ggv, x, ggx, A1, nullptr);
  return cudaGetLastError();
}

template <int RM, int LF>
cudaError_t launch_wn_dbls(const DevPlan& d, int s0, int nc, const int* s_rowptr, const int* perm,
                           const int* s_recv, const float* vec, const float* ggv, const float* g, float* B1,
                           float* B0, cudaStream_t st) {
  if (nc <= 0) return cudaSuccess;
  if (B0)
    k_wn_stream<RM, LF, 1, false, true, true><<<wn_grid_pm(d, nc), 32 * kWnWarps, d.wn_smem_s2, st>>>(
        d, s0, nc, s_rowptr, s_recv, perm, vec, ggv, g, nullptr, B1, B0);
  else
    k_wn_stream<RM, LF, 1, false, true, false><<<wn_grid_pm(d, nc), 32 * kWnWarps, d.wn_smem_s2, st>>>(
        d, s0, nc, s_rowptr, s_recv, perm, vec, ggv, g, nullptr, B1, nullptr);
  return cudaGetLastError();
}

template <int RM, int LF>
cudaError_t launch_wn_adj(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                          const float* x, const float* G, float* dvec, float* dY, float* db, cudaStream_t st) {
  if (nc <= 0) return cudaSuccess;
  k_wn_adj<RM, LF, false, false><<<wn_grid(nc), 32 * kWnWarps, d.wn_smem_adj, st>>>(
      d, r0, nc, rowptr, col, vec, nullptr, x, nullptr, G, nullptr, dvec, dY, db);
  return cudaGetLastError();
}

template <int RM, int LF>
cudaError_t launch_wn_dadj(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                           const float* ggv, const float* x, const float* ggx, const float* G, const float* Gt,
                           float* dvec, cudaStream_t st) {
  if (nc <= 0) return cudaSuccess;
  if (Gt)
    k_wn_adj<RM, LF, true, true><<<wn_grid(nc), 32 * kWnWarps, d.wn_smem_dadj, st>>>(
        d, r0, nc, rowptr, col, vec, ggv, x, ggx, G, Gt, dvec, nullptr, nullptr);
  else
    k_wn_adj<RM, LF, true, false><<<wn_grid(nc), 32 * kWnWarps, d.wn_smem_dadj, st>>>(
        d, r0, nc, rowptr, col, vec, ggv, x, ggx, G, nullptr, dvec, nullptr, nullptr);
  return cudaGetLastError();
}

}  // namespace tpc

// One translation unit per kernel instantiation keeps the parallel build even.
#define TPC_WN_TU_CPL(tag, form, RM, LF, CPL, RECV, DBL, ...)                 \
  namespace tpc {                                                             \
  template cudaError_t launch_wn_##form<RM, LF, CPL>(__VA_ARGS__);            \
  }                                                                           \
  TPC_REGISTER_TU(tag, (&tpc::wn_smem<RM, LF, CPL, RECV, DBL>))
#define TPC_WN_TU(tag, form, RM, LF, RECV, DBL, ...)                          \
  namespace tpc {                                                             \
  template cudaError_t launch_wn_##form<RM, LF>(__VA_ARGS__);                 \
  }                                                                           \
  TPC_REGISTER_TU(tag, (&tpc::wn_smem<RM, LF, 1, RECV, DBL>))
#define TPC_WNA_TU(tag, form, RM, LF, DBL, ...)                               \
  namespace tpc {                                                             \
  template cudaError_t launch_wn_##form<RM, LF>(__VA_ARGS__);                 \
  }                                                                           \
  TPC_REGISTER_TU(tag, (&tpc::wna_smem<RM, LF, DBL>))
