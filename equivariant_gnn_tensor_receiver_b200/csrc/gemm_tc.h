// Tensor-core (tcgen05) GEMM for the node-level Theta contraction.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace tpc {

// C(i, j) = p[(i / rdiv) * r_hi + (i % rdiv) * r_lo + j * c_hi]
struct TcOut {
  float* p;
  int64_t rdiv, r_hi, r_lo, c_hi;
};

// Per-context set-up: the kernels' dynamic shared-memory limits.
cudaError_t gemm_tc_init();

// TMA / descriptor requirements: 16-byte aligned bases, row pitches a multiple of 4 floats.
bool gemm_tc_supported(const float* A, int64_t lda, const float* B, int64_t ldb, int M, int N, int K);

// C (+)= A[M][K] . B[N][K]^T.  split = 3xTF32 (B and Blo precomputed), else one TF32 pass.
// limit: nanoseconds any wait on the kernel's own pipeline may take before the
// kernel records an error (gemm_tc_read_error) and gives up.
constexpr uint64_t kDefaultWaitNs = 2000000000ull;
cudaError_t gemm_tc(const float* A, int64_t lda, const float* B, const float* Blo, int64_t ldb, int M, int N, int K,
                    TcOut out, int accumulate, bool split, cudaStream_t st, uint64_t limit = kDefaultWaitNs);

// Theta block [K][N] -> hi = its transpose [N][K] (rounded to TF32 when lo != null), lo = remainder.
cudaError_t split_transpose(const float* th, int K, int N, float* hi, float* lo, cudaStream_t st);

// hi = rn_tf32(v), lo = rn_tf32(v - hi) elementwise (lo null: plain copy)
cudaError_t split_elementwise(const float* v, int64_t n, float* hi, float* lo, cudaStream_t st);

// Theta[p] ([R][c_in][c_out]) of every listed path into columns kxoff + k*c_out + w of its [c_in][Kx]
// matrix at dst_off (split when lo != null), all paths in one launch
struct XPackPath {
  int64_t theta_off, dst_off;
  int c_in, c_out, kxoff, Kx;
};
constexpr int kXPackMax = 48;
struct XPackList {
  int n, R;
  XPackPath p[kXPackMax];
};
cudaError_t theta_x_pack_all(const float* th, const XPackList& l, float* hi, float* lo, cudaStream_t st);

// rows (node, m) x columns w of one feature block of nodes r0 : r0+nc -> dense [nc*n3][mul]
cudaError_t pack_rows(const float* g, int dim, int off, int mul, int n3, int64_t r0, int nc, float* out,
                      cudaStream_t st);

// First error code recorded by an expired wait of a tensor-core GEMM since the
// last read (0 = none); clears it.  The caller synchronises first.
cudaError_t gemm_tc_read_error(int* code);

}  // namespace tpc
