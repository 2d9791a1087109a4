// Launchers of the edge-lane (receiver adjoint) warp-per-node streams
// (instantiated per (RM, LF) in tu_wn_{adj,dadj}_*.cu).
#pragma once

#include "launch_streams.cuh"
#include "launch_wn_common.cuh"
#include "streams_wna.cuh"

namespace tpc {

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

template <int RM, int LF>
cudaError_t launch_wn_adj(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                          const float* x, const float* G, float* dvec, float* dY, float* db, const int* extra,
                          int* counter, cudaStream_t st) {
  if (nc <= 0) return cudaSuccess;
  auto k = k_wn_adj<RM, LF, false, false>;
  k<<<wn_grid(k, d.wn_smem_adj), 32 * kWnWarps, d.wn_smem_adj, st>>>(d, r0, nc, rowptr, col, vec, nullptr, x, nullptr,
                                                                      G, nullptr, dvec, dY, db, extra, counter);
  return cudaGetLastError();
}

// Second order with l = 3 features runs one CTA per SM: its G staging reads a
// cache line of G across eight channel chunks, and with a second CTA's shared
// memory the SM has no L1 left to keep those lines (measured on the wide layer,
// 128 channels per block up to l = 3: 45 ms with two CTAs per SM, 27 ms with one).
template <int LF>
int dadj_smem(int bytes) {
  return LF >= 3 ? std::max(bytes, kWnaTwoCtaBytes + 1024) : bytes;
}

template <int RM, int LF>
cudaError_t launch_wn_dadj(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                           const float* ggv, const float* x, const float* ggx, const float* G, const float* Gt,
                           float* dvec, const int* extra, int* counter, cudaStream_t st) {
  if (nc <= 0) return cudaSuccess;
  if (Gt) {
    auto k = k_wn_adj<RM, LF, true, true>;
    const int smem = dadj_smem<LF>(wna_smem_bytes(d.rm, d.n3max, d.n1max, true, true));
    k<<<wn_grid(k, smem), 32 * kWnWarps, smem, st>>>(d, r0, nc, rowptr, col, vec, ggv, x, ggx, G, Gt, dvec, nullptr,
                                                     nullptr, extra, counter);
  } else {
    auto k = k_wn_adj<RM, LF, true, false>;
    const int smem = dadj_smem<LF>(d.wn_smem_dadj);
    k<<<wn_grid(k, smem), 32 * kWnWarps, smem, st>>>(d, r0, nc, rowptr, col, vec, ggv, x, ggx, G, nullptr, dvec,
                                                     nullptr, nullptr, extra, counter);
  }
  return cudaGetLastError();
}

}  // namespace tpc

#define TPC_WNA_TU(tag, form, RM, LF, DBL, ...)                               \
  namespace tpc {                                                             \
  template cudaError_t launch_wn_##form<RM, LF>(__VA_ARGS__);                 \
  }                                                                           \
  TPC_REGISTER_TU(tag, (&tpc::wna_smem<RM, LF, DBL>))
