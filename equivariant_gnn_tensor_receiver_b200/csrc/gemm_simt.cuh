// Plain fp32 FFMA GEMM over strided operand views: the node-level Theta
// contractions of the streaming schedule in reference precision.  Every
// operand element (i, j) lives at
//     p[(i / rdiv) * r_hi + (i % rdiv) * r_lo + (j / cdiv) * c_hi + (j % cdiv) * c_lo],
// which expresses the feature layouts ([node][mul][2l+1]) directly, so no
// repacking is needed.  C = A B (overwrite), C += A B, or split-K with atomic
// accumulation into a zeroed C.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

namespace tpc {

struct MView {
  float* p;
  int64_t rdiv, r_hi, r_lo;
  int64_t cdiv, c_hi, c_lo;
};

__host__ __device__ inline MView mview(float* p, int64_t rdiv, int64_t r_hi, int64_t r_lo, int64_t cdiv,
                                       int64_t c_hi, int64_t c_lo) {
  MView v;
  v.p = p;
  v.rdiv = rdiv;
  v.r_hi = r_hi;
  v.r_lo = r_lo;
  v.cdiv = cdiv;
  v.c_hi = c_hi;
  v.c_lo = c_lo;
  return v;
}
// plain row-major matrix with leading dimension ld
__host__ __device__ inline MView mrow(float* p, int64_t ld) { return mview(p, 1, ld, 0, 1, 1, 0); }

__device__ __forceinline__ int64_t maddr(const MView& v, int64_t i, int64_t j) {
  return (i / v.rdiv) * v.r_hi + (i % v.rdiv) * v.r_lo + (j / v.cdiv) * v.c_hi + (j % v.cdiv) * v.c_lo;
}

constexpr int kGemmBM = 64, kGemmBN = 64, kGemmBK = 16;

// mode: 0 overwrite, 1 accumulate, 2 atomic accumulate (split-K)
__global__ void __launch_bounds__(256) k_gemm_simt(int64_t M, int64_t N, int64_t K, MView A, MView B,
                                                   MView C, int mode, int64_t k_per_split) {
  __shared__ float sA[kGemmBK][kGemmBM + 4];
  __shared__ float sB[kGemmBK][kGemmBN + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t m0 = int64_t(blockIdx.x) * kGemmBM, n0 = int64_t(blockIdx.y) * kGemmBN;
  const int64_t kb = int64_t(blockIdx.z) * k_per_split;
  const int64_t ke = min(K, kb + k_per_split);
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int64_t k0 = kb; k0 < ke; k0 += kGemmBK) {
    for (int t = threadIdx.x; t < kGemmBK * kGemmBM; t += 256) {
      const int kk = t / kGemmBM, mm = t % kGemmBM;
      const int64_t gm = m0 + mm, gk = k0 + kk;
      sA[kk][mm] = (gm < M && gk < ke) ? A.p[maddr(A, gm, gk)] : 0.f;
    }
    for (int t = threadIdx.x; t < kGemmBK * kGemmBN; t += 256) {
      const int kk = t / kGemmBN, nn = t % kGemmBN;
      const int64_t gn = n0 + nn, gk = k0 + kk;
      sB[kk][nn] = (gn < N && gk < ke) ? B.p[maddr(B, gk, gn)] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kGemmBK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = sA[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = sB[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t gm = m0 + ty + 16 * i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t gn = n0 + tx + 16 * j;
      if (gn >= N) continue;
      float* c = C.p + maddr(C, gm, gn);
      if (mode == 0) *c = acc[i][j];
      else if (mode == 1) *c += acc[i][j];
      else atomicAdd(c, acc[i][j]);
    }
  }
}

inline cudaError_t gemm_simt(int64_t M, int64_t N, int64_t K, MView A, MView B, MView C, int mode,
                             cudaStream_t st) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  int64_t tiles = ((M + kGemmBM - 1) / kGemmBM) * ((N + kGemmBN - 1) / kGemmBN);
  int64_t splits = 1;
  if (mode == 2) {
    // enough CTAs to fill the GPU, each with at least 256 of K
    splits = std::max<int64_t>(1, std::min<int64_t>((K + 255) / 256, (4 * 148 + tiles - 1) / tiles));
  }
  int64_t kps = (K + splits - 1) / splits;
  kps = (kps + kGemmBK - 1) / kGemmBK * kGemmBK;
  if (kps == 0) kps = kGemmBK;
  splits = K > 0 ? (K + kps - 1) / kps : 1;
  dim3 grid(unsigned((M + kGemmBM - 1) / kGemmBM), unsigned((N + kGemmBN - 1) / kGemmBN), unsigned(splits));
  k_gemm_simt<<<grid, 256, 0, st>>>(M, N, K, A, B, C, mode, kps);
  return cudaGetLastError();
}

}  // namespace tpc
