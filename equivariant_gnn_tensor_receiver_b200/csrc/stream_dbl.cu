// Double-backward edge streams: per-path receiver / sender streams and the fused
// adjoint stream.
#include <algorithm>

#include "launchers.h"
#include "streams_dbl.cuh"

namespace tpc {

TPC_DEFINE_CG_UPLOADER(upload_cg_dbl)

cudaError_t dbl_set_smem_limit(int bytes) {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(k_dbl_r_stream<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes))) return e;
  if ((e = cudaFuncSetAttribute(k_dbl_r_stream<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes))) return e;
  return cudaFuncSetAttribute(k_dbl_r_stream<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <int RM>
static cudaError_t dbl_a_one(const DevPlan& d, int p, int r0, int nc, const int* rowptr, const int* col,
                             const float* vec, const float* ggv, const float* x, const float* ggx, float* A1,
                             float* A0, cudaStream_t st) {
  const DevPath& q = d.path[p];
  dim3 grid(unsigned((nc + kWarpsPerBlock - 1) / kWarpsPerBlock), unsigned((q.c_in + 31) / 32));
  switch (triple_id(q.l1, q.l2, q.l3)) {
#define TPC_CASE(a, b, c)                                                                                    \
  case triple_id(a, b, c):                                                                                   \
    k_dbl_a_path<a, b, c, RM><<<grid, 32 * kWarpsPerBlock, 0, st>>>(d, p, r0, nc, rowptr, col, vec, ggv, x, \
                                                                    ggx, A1, A0);                            \
    break;
    TPC_FOR_EACH_TRIPLE(TPC_CASE)
#undef TPC_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <int RM>
static cudaError_t dbl_s_one(const DevPlan& d, int p, int s0, int nc, const int* s_rowptr, const int* perm,
                             const int* s_recv, const float* vec, const float* ggv, const float* g, float* B1,
                             float* B0, cudaStream_t st) {
  const DevPath& q = d.path[p];
  dim3 grid(unsigned((nc + kWarpsPerBlock - 1) / kWarpsPerBlock), unsigned((q.c_out + 31) / 32));
  switch (triple_id(q.l1, q.l2, q.l3)) {
#define TPC_CASE(a, b, c)                                                                                      \
  case triple_id(a, b, c):                                                                                     \
    k_dbl_s_path<a, b, c, RM><<<grid, 32 * kWarpsPerBlock, 0, st>>>(d, p, s0, nc, s_rowptr, perm, s_recv, vec, \
                                                                    ggv, g, B1, B0);                           \
    break;
    TPC_FOR_EACH_TRIPLE(TPC_CASE)
#undef TPC_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_dbl_a_stream(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col,
                                const float* vec, const float* ggv, const float* x, const float* ggx, float* A1,
                                float* A0, cudaStream_t st) {
  for (int p = 0; p < d.P; ++p) {
    cudaError_t e;
    if (d.rm == 4) e = dbl_a_one<4>(d, p, r0, nc, rowptr, col, vec, ggv, x, ggx, A1, A0, st);
    else if (d.rm == 8) e = dbl_a_one<8>(d, p, r0, nc, rowptr, col, vec, ggv, x, ggx, A1, A0, st);
    else e = dbl_a_one<16>(d, p, r0, nc, rowptr, col, vec, ggv, x, ggx, A1, A0, st);
    if (e) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_dbl_s_stream(const DevPlan& d, int s0, int nc, const int* s_rowptr, const int* perm,
                                const int* s_recv, const float* vec, const float* ggv, const float* g, float* B1,
                                float* B0, cudaStream_t st) {
  for (int p = 0; p < d.P; ++p) {
    cudaError_t e;
    if (d.rm == 4) e = dbl_s_one<4>(d, p, s0, nc, s_rowptr, perm, s_recv, vec, ggv, g, B1, B0, st);
    else if (d.rm == 8) e = dbl_s_one<8>(d, p, s0, nc, s_rowptr, perm, s_recv, vec, ggv, g, B1, B0, st);
    else e = dbl_s_one<16>(d, p, s0, nc, s_rowptr, perm, s_recv, vec, ggv, g, B1, B0, st);
    if (e) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_dbl_r_stream(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col,
                                const float* vec, const float* ggv, const float* x, const float* ggx,
                                const float* G, const float* Gt, float* dvec, cudaStream_t st) {
  const int threads = 32 * std::min(d.P, 16);
  const size_t smem = size_t(d.sm_floats2) * 4;
  if (d.rm == 4)
    k_dbl_r_stream<4><<<unsigned(nc), threads, smem, st>>>(d, r0, nc, rowptr, col, vec, ggv, x, ggx, G, Gt, dvec);
  else if (d.rm == 8)
    k_dbl_r_stream<8><<<unsigned(nc), threads, smem, st>>>(d, r0, nc, rowptr, col, vec, ggv, x, ggx, G, Gt, dvec);
  else
    k_dbl_r_stream<16><<<unsigned(nc), threads, smem, st>>>(d, r0, nc, rowptr, col, vec, ggv, x, ggx, G, Gt,
                                                            dvec);
  return cudaGetLastError();
}

}  // namespace tpc
