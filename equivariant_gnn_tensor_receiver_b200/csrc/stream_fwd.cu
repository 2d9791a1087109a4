// Forward receiver stream: one kernel instantiation per (CG triple, radial width).
#include "launchers.h"
#include "streams.cuh"

namespace tpc {

TPC_DEFINE_CG_UPLOADER(upload_cg_fwd)

template <int RM>
static cudaError_t fwd_one(const DevPlan& d, int p, int r0, int nc, const int* rowptr, const int* col,
                           const float* vec, const float* x, float* A, cudaStream_t st) {
  const DevPath& q = d.path[p];
  dim3 grid(unsigned((nc + kWarpsPerBlock - 1) / kWarpsPerBlock), unsigned((q.c_in + 31) / 32));
  switch (triple_id(q.l1, q.l2, q.l3)) {
#define TPC_CASE(a, b, c)                                                                          \
  case triple_id(a, b, c):                                                                         \
    k_fwd_path<a, b, c, RM><<<grid, 32 * kWarpsPerBlock, 0, st>>>(d, p, r0, nc, rowptr, col, vec, x, A); \
    break;
    TPC_FOR_EACH_TRIPLE(TPC_CASE)
#undef TPC_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_fwd_stream(const DevPlan& d, int r0, int nc, const int* rowptr, const int* col,
                              const float* vec, const float* x, float* A, cudaStream_t st) {
  for (int p = 0; p < d.P; ++p) {
    cudaError_t e;
    if (d.rm == 4) e = fwd_one<4>(d, p, r0, nc, rowptr, col, vec, x, A, st);
    else if (d.rm == 8) e = fwd_one<8>(d, p, r0, nc, rowptr, col, vec, x, A, st);
    else e = fwd_one<16>(d, p, r0, nc, rowptr, col, vec, x, A, st);
    if (e) return e;
  }
  return cudaSuccess;
}

}  // namespace tpc
