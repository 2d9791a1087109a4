// Launchers of the channel-lane warp-per-node edge streams (instantiated per
// (RM, LF[, CPL]) in tu_wn_{fwd,send,dbla,dbls}_*.cu).  One warp per node of the
// chunk, kWnWarps nodes per CTA.
#pragma once

#include "launch_streams.cuh"
#include "launch_wn_common.cuh"
#include "streams_wn.cuh"

namespace tpc {

template <int RM, int LF, int CPL, bool RECV, bool DBL>
cudaError_t wn_smem(int bytes) {
  const auto attr = cudaFuncAttributeMaxDynamicSharedMemorySize;
  cudaError_t e = cudaFuncSetAttribute(k_wn_stream<RM, LF, CPL, RECV, DBL, false, false>, attr, bytes);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(k_wn_stream<RM, LF, CPL, RECV, DBL, false, true>, attr, bytes);
  if constexpr (DBL) {
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k_wn_stream<RM, LF, CPL, RECV, true, true, false>, attr, bytes);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k_wn_stream<RM, LF, CPL, RECV, true, true, true>, attr, bytes);
  }
  return e;
}
template <int RM, int LF, int CPL>
cudaError_t launch_wn_fwd(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                          const float* x, float* A, const int* extra, int* counter, int seg, cudaStream_t st) {
  if (nc <= 0) return cudaSuccess;
  auto k = k_wn_stream<RM, LF, CPL, true, false, false, false>;
  auto kx = k_wn_stream<RM, LF, CPL, true, false, false, true>;
  k<<<wn_grid_pm(d, nc), 32 * kWnWarps, d.wn_smem_f, st>>>(d, r0, nc, rowptr, col, nullptr, vec, nullptr, x,
                                                                  nullptr, A, nullptr, extra, counter, seg);
  kx<<<wn_grid(kx, d.wn_smem_f), 32 * kWnWarps, d.wn_smem_f, st>>>(d, r0, nc, rowptr, col, nullptr, vec, nullptr, x,
                                                                  nullptr, A, nullptr, extra, counter, seg);
  return cudaGetLastError();
}

template <int RM, int LF, int CPL>
cudaError_t launch_wn_send(const DevPlan& d, int s0, int nc, const int* s_rowptr, const int* perm,
                           const int* s_recv, const float* vec, const float* g, float* B, const int* extra,
                           int* counter, int seg, cudaStream_t st) {
  if (nc <= 0) return cudaSuccess;
  auto k = k_wn_stream<RM, LF, CPL, false, false, false, false>;
  auto kx = k_wn_stream<RM, LF, CPL, false, false, false, true>;
  k<<<wn_grid_pm(d, nc), 32 * kWnWarps, d.wn_smem_s, st>>>(d, s0, nc, s_rowptr, s_recv, perm, vec, nullptr, g,
                                                                  nullptr, B, nullptr, extra, counter, seg);
  kx<<<wn_grid(kx, d.wn_smem_s), 32 * kWnWarps, d.wn_smem_s, st>>>(d, s0, nc, s_rowptr, s_recv, perm, vec, nullptr, g,
                                                                  nullptr, B, nullptr, extra, counter, seg);
  return cudaGetLastError();
}

template <int RM, int LF>
cudaError_t launch_wn_dbla(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                           const float* ggv, const float* x, const float* ggx, float* A1, float* A0,
                           const int* extra, int* counter, int seg, cudaStream_t st) {
  if (nc <= 0) return cudaSuccess;
  if (A0) {
    auto k = k_wn_stream<RM, LF, 1, true, true, true, false>;
    auto kx = k_wn_stream<RM, LF, 1, true, true, true, true>;
    k<<<wn_grid_pm(d, nc), 32 * kWnWarps, d.wn_smem_f2, st>>>(d, r0, nc, rowptr, col, nullptr, vec, ggv, x,
                                                                      ggx, A1, A0, extra, counter, seg);
    kx<<<wn_grid(kx, d.wn_smem_f2), 32 * kWnWarps, d.wn_smem_f2, st>>>(d, r0, nc, rowptr, col, nullptr, vec, ggv, x,
                                                                      ggx, A1, A0, extra, counter, seg);
  } else {
    auto k = k_wn_stream<RM, LF, 1, true, true, false, false>;
    auto kx = k_wn_stream<RM, LF, 1, true, true, false, true>;
    k<<<wn_grid_pm(d, nc), 32 * kWnWarps, d.wn_smem_f2, st>>>(d, r0, nc, rowptr, col, nullptr, vec, ggv, x,
                                                                      ggx, A1, nullptr, extra, counter, seg);
    kx<<<wn_grid(kx, d.wn_smem_f2), 32 * kWnWarps, d.wn_smem_f2, st>>>(d, r0, nc, rowptr, col, nullptr, vec, ggv, x,
                                                                      ggx, A1, nullptr, extra, counter, seg);
  }
  return cudaGetLastError();
}

template <int RM, int LF>
cudaError_t launch_wn_dbls(const DevPlan& d, int s0, int nc, const int* s_rowptr, const int* perm,
                           const int* s_recv, const float* vec, const float* ggv, const float* g, float* B1,
                           float* B0, const int* extra, int* counter, int seg, cudaStream_t st) {
  if (nc <= 0) return cudaSuccess;
  if (B0) {
    auto k = k_wn_stream<RM, LF, 1, false, true, true, false>;
    auto kx = k_wn_stream<RM, LF, 1, false, true, true, true>;
    k<<<wn_grid_pm(d, nc), 32 * kWnWarps, d.wn_smem_s2, st>>>(d, s0, nc, s_rowptr, s_recv, perm, vec, ggv, g,
                                                                      nullptr, B1, B0, extra, counter, seg);
    kx<<<wn_grid(kx, d.wn_smem_s2), 32 * kWnWarps, d.wn_smem_s2, st>>>(d, s0, nc, s_rowptr, s_recv, perm, vec, ggv, g,
                                                                      nullptr, B1, B0, extra, counter, seg);
  } else {
    auto k = k_wn_stream<RM, LF, 1, false, true, false, false>;
    auto kx = k_wn_stream<RM, LF, 1, false, true, false, true>;
    k<<<wn_grid_pm(d, nc), 32 * kWnWarps, d.wn_smem_s2, st>>>(d, s0, nc, s_rowptr, s_recv, perm, vec, ggv, g,
                                                                      nullptr, B1, nullptr, extra, counter, seg);
    kx<<<wn_grid(kx, d.wn_smem_s2), 32 * kWnWarps, d.wn_smem_s2, st>>>(d, s0, nc, s_rowptr, s_recv, perm, vec, ggv, g,
                                                                      nullptr, B1, nullptr, extra, counter, seg);
  }
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
