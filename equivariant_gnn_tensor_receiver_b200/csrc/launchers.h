// Host-side launchers of the edge-stream kernels.  Each kernel family is
// instantiated per radial register width RM (8, 16) in its own translation
// unit (tu_*.cu); every unit registers an initialiser that uploads its copy of
// the constant CG table and raises its kernels' shared-memory limit.
#pragma once

#include <cuda_runtime.h>

#include <vector>

#include "plan.h"

namespace tpc {

struct TuInit {
  cudaError_t (*upload)(const float* table);  // this unit's __constant__ CG table
  cudaError_t (*smem)(int bytes);             // dynamic shared memory limits (may be null)
};
std::vector<TuInit>& tu_registry();
struct TuRegistrar {
  explicit TuRegistrar(TuInit t) { tu_registry().push_back(t); }
};

// backward: per-edge dvec / dY / db of receivers r0 : r0+nc from G of the chunk
// (per-path stream, for plans whose rows cannot be staged 16 bytes at a time)
template <int RM>
cudaError_t launch_radj_rm(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                           const float* x, const float* G, float* dvec, float* dY, float* db, cudaStream_t st);
// double backward: d_vec of receivers r0 : r0+nc from G (and Gt, may be null)
template <int RM>
cudaError_t launch_dbl_r_rm(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                            const float* ggv, const float* x, const float* ggx, const float* G, const float* Gt,
                            float* dvec, cudaStream_t st);

// Warp-per-node streams (streams_wn.cuh, streams_wna.cuh), one warp per node.
// LF bounds the feature degrees l1, l3 of the paths the kernel handles; CPL is
// the number of channels per lane of the channel-lane forms.
template <int RM, int LF, int CPL>
cudaError_t launch_wn_fwd(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                          const float* x, float* A, const int* extra, int* counter, int seg, cudaStream_t st);
template <int RM, int LF, int CPL>
cudaError_t launch_wn_send(const DevPlan& d, int s0, int nc, const int* s_rowptr, const int* perm,
                           const int* s_recv, const float* vec, const float* g, float* B, const int* extra,
                           int* counter, int seg, cudaStream_t st);
template <int RM, int LF>
cudaError_t launch_wn_dbla(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                           const float* ggv, const float* x, const float* ggx, float* A1, float* A0,
                           const int* extra, int* counter, int seg, cudaStream_t st);
template <int RM, int LF>
cudaError_t launch_wn_dbls(const DevPlan& d, int s0, int nc, const int* s_rowptr, const int* perm,
                           const int* s_recv, const float* vec, const float* ggv, const float* g, float* B1,
                           float* B0, const int* extra, int* counter, int seg, cudaStream_t st);
template <int RM, int LF>
cudaError_t launch_wn_adj(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                          const float* x, const float* G, float* dvec, float* dY, float* db, const int* extra,
                          int* counter, cudaStream_t st);
template <int RM, int LF>
cudaError_t launch_wn_dadj(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                           const float* ggv, const float* x, const float* ggx, const float* G, const float* Gt,
                           float* dvec, const int* extra, int* counter, cudaStream_t st);

// instantiation of a warp-per-node launcher for the plan's (rm, wn_lf[, wn_cpl])
#define TPC_WN_CALL(d, fn, ...) \
  ((d).rm == 16 ? fn<16, 3>(__VA_ARGS__) : (d).wn_lf == 2 ? fn<8, 2>(__VA_ARGS__) : fn<8, 3>(__VA_ARGS__))
#define TPC_WN_CALL_CPL(d, fn, ...)                                                                     \
  ((d).rm == 16      ? fn<16, 3, 1>(__VA_ARGS__)                                                        \
   : (d).wn_lf == 2 ? ((d).wn_cpl == 2 ? fn<8, 2, 2>(__VA_ARGS__) : fn<8, 2, 1>(__VA_ARGS__))           \
                    : fn<8, 3, 1>(__VA_ARGS__))

#define TPC_RM_CALL(rm, fn, ...) ((rm) == 8 ? fn<8>(__VA_ARGS__) : fn<16>(__VA_ARGS__))

}  // namespace tpc
