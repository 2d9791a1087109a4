// Host-side launchers of the edge-stream kernels.  Each kernel family is
// instantiated per radial register width RM (4, 8, 16) in its own translation
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

// forward: A[r0 : r0+nc] for every path (receiver-sorted)
template <int RM>
cudaError_t launch_fwd_rm(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                          const float* x, float* A, cudaStream_t st);
// backward: B[s0 : s0+nc] for every path (sender-sorted)
template <int RM>
cudaError_t launch_send_rm(const DevPlan& d, int s0, int nc, const int* s_rowptr, const int* perm,
                           const int* s_recv, const float* vec, const float* g, float* B, cudaStream_t st);
// backward: per-edge dvec / dY / db of receivers r0 : r0+nc from G of the chunk
template <int RM>
cudaError_t launch_radj_rm(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                           const float* x, const float* G, float* dvec, float* dY, float* db, cudaStream_t st);
// backward, lane-per-edge variant (requires plan.adj_cw > 0)
template <int RM>
cudaError_t launch_adj_rm(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                          const float* x, const float* G, float* dvec, float* dY, float* db, cudaStream_t st);
// double backward, lane-per-edge adjoint stream (requires plan.dadj_cw > 0)
template <int RM>
cudaError_t launch_dadj_rm(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                           const float* ggv, const float* x, const float* ggx, const float* G, const float* Gt,
                           float* dvec, cudaStream_t st);
// double backward: [A1 | A0] of receivers r0 : r0+nc
template <int RM>
cudaError_t launch_dbl_a_rm(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                            const float* ggv, const float* x, const float* ggx, float* A1, float* A0,
                            cudaStream_t st);
// double backward: [B1 | B0] of senders s0 : s0+nc
template <int RM>
cudaError_t launch_dbl_s_rm(const DevPlan& d, int s0, int nc, const int* s_rowptr, const int* perm,
                            const int* s_recv, const float* vec, const float* ggv, const float* g, float* B1,
                            float* B0, cudaStream_t st);
// double backward: d_vec of receivers r0 : r0+nc from G (and Gt, may be null)
template <int RM>
cudaError_t launch_dbl_r_rm(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col, const float* vec,
                            const float* ggv, const float* x, const float* ggx, const float* G, const float* Gt,
                            float* dvec, cudaStream_t st);

#define TPC_RM_CALL(rm, fn, ...) \
  ((rm) == 4 ? fn<4>(__VA_ARGS__) : (rm) == 8 ? fn<8>(__VA_ARGS__) : fn<16>(__VA_ARGS__))

}  // namespace tpc
