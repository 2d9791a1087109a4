// Host-side launchers of the edge-stream kernels (one translation unit each).
#pragma once

#include <cuda_runtime.h>

#include "plan.h"

namespace tpc {

cudaError_t upload_cg_fwd(const float* table);
cudaError_t upload_cg_send(const float* table);
cudaError_t upload_cg_radj(const float* table);
cudaError_t upload_cg_dbl(const float* table);
cudaError_t radj_set_smem_limit(int bytes);
cudaError_t dbl_set_smem_limit(int bytes);

// A[r0 : r0+nc] for every path (receiver-sorted forward stream)
cudaError_t launch_fwd_stream(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col,
                              const float* vec, const float* x, float* A, cudaStream_t st);
// B[s0 : s0+nc] for every path (sender-sorted backward stream)
cudaError_t launch_send_stream(const DevPlan& d, int s0, int nc, const int* s_rowptr, const int* perm,
                               const int* s_recv, const float* vec, const float* g, float* B, cudaStream_t st);
// per-edge dvec / dY / db of the receivers r0 : r0+nc, from G of the same chunk
cudaError_t launch_radj_stream(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col,
                               const float* vec, const float* x, const float* G, float* dvec, float* dY,
                               float* db, cudaStream_t st);

// double backward: [A1 | A0] of receivers r0 : r0+nc
cudaError_t launch_dbl_a_stream(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col,
                                const float* vec, const float* ggv, const float* x, const float* ggx, float* A1,
                                float* A0, cudaStream_t st);
// double backward: [B1 | B0] of senders s0 : s0+nc
cudaError_t launch_dbl_s_stream(const DevPlan& d, int s0, int nc, const int* s_rowptr, const int* perm,
                                const int* s_recv, const float* vec, const float* ggv, const float* g, float* B1,
                                float* B0, cudaStream_t st);
// double backward: d_vec of the receivers r0 : r0+nc from G (and Gt, may be null)
cudaError_t launch_dbl_r_stream(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col,
                                const float* vec, const float* ggv, const float* x, const float* ggx,
                                const float* G, const float* Gt, float* dvec, cudaStream_t st);

}  // namespace tpc
