// Backward sender stream: one kernel instantiation per (CG triple, radial width).
#include "launchers.h"
#include "streams.cuh"

namespace tpc {

TPC_DEFINE_CG_UPLOADER(upload_cg_send)

template <int RM>
static cudaError_t send_one(const DevPlan& d, int p, int s0, int nc, const int* s_rowptr, const int* perm,
                            const int* s_recv, const float* vec, const float* g, float* B, cudaStream_t st) {
  const DevPath& q = d.path[p];
  dim3 grid(unsigned((nc + kWarpsPerBlock - 1) / kWarpsPerBlock), unsigned((q.c_out + 31) / 32));
  switch (triple_id(q.l1, q.l2, q.l3)) {
#define TPC_CASE(a, b, c)                                                                        \
  case triple_id(a, b, c):                                                                       \
    k_send_path<a, b, c, RM><<<grid, 32 * kWarpsPerBlock, 0, st>>>(d, p, s0, nc, s_rowptr, perm, \
                                                                   s_recv, vec, g, B);           \
    break;
    TPC_FOR_EACH_TRIPLE(TPC_CASE)
#undef TPC_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_send_stream(const DevPlan& d, int s0, int nc, const int* s_rowptr, const int* perm,
                               const int* s_recv, const float* vec, const float* g, float* B, cudaStream_t st) {
  for (int p = 0; p < d.P; ++p) {
    cudaError_t e;
    if (d.rm == 4) e = send_one<4>(d, p, s0, nc, s_rowptr, perm, s_recv, vec, g, B, st);
    else if (d.rm == 8) e = send_one<8>(d, p, s0, nc, s_rowptr, perm, s_recv, vec, g, B, st);
    else e = send_one<16>(d, p, s0, nc, s_rowptr, perm, s_recv, vec, g, B, st);
    if (e) return e;
  }
  return cudaSuccess;
}

}  // namespace tpc
