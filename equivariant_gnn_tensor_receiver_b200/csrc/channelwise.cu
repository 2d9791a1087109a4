// Node-level contractions of the channel-wise operator family (see channelwise.h).
//
// Every kernel runs 32 x 8 thread blocks: x spans 32 consecutive channels (or
// state columns), so each row of A / G / B is read or written as whole 128-byte
// lines; y spans nodes of the chunk, grid-strided.  The grid holds about eight
// blocks per SM.  Theta is a few KB and stays in L1.
#include <cuda_runtime.h>

#include <algorithm>

#include "channelwise.h"

namespace tpc {
namespace {

constexpr int kTX = 32, kTY = 8;
constexpr int kTargetBlocks = 148 * 8;

dim3 cw_grid(int nc, int cols) {
  const int gy = (cols + kTX - 1) / kTX;
  const int gx = std::max(1, std::min((nc + kTY - 1) / kTY, std::max(1, kTargetBlocks / gy)));
  return dim3(unsigned(gx), unsigned(gy));
}

// column j of a block's state -> (path, radial index, channel); path -1 if none
__device__ __forceinline__ int cw_column(const DevPlan& d, bool recv, int blk, int j, int* k, int* u) {
  for (int p = 0; p < d.P; ++p) {
    const DevPath& q = d.path[p];
    if ((recv ? q.i3 : q.i1) != blk) continue;
    const int off = recv ? q.koff : q.kxoff, c = q.c_in;
    if (j >= off && j < off + d.R * c) {
      *k = (j - off) / c;
      *u = j - off - *k * c;
      return p;
    }
  }
  return -1;
}

__global__ void __launch_bounds__(kTX* kTY) k_cw_forward(const __grid_constant__ DevPlan d, int i3, int r0, int nc,
                                                         const float* __restrict__ A,
                                                         const float* __restrict__ theta, float* __restrict__ out,
                                                         int mode) {
  const int c = d.out_mul[i3], n3 = 2 * d.out_l[i3] + 1, Kb = d.Kb[i3];
  const int u = blockIdx.y * kTX + threadIdx.x;
  if (u >= c) return;
  int p0 = 0;  // paths are ordered by output block: [p0, p1) feed i3
  while (p0 < d.P && d.path[p0].i3 != i3) ++p0;
  int p1 = p0;
  while (p1 < d.P && d.path[p1].i3 == i3) ++p1;
  const float* Ab = A + size_t(nc) * d.a_pref[i3] + u;
  for (int n = blockIdx.x * kTY + threadIdx.y; n < nc; n += gridDim.x * kTY) {
    float* o = out + size_t(r0 + n) * d.dim_out + d.out_off[i3] + u * n3;
    for (int m3 = 0; m3 < n3; ++m3) {
      const float* a = Ab + (size_t(n) * n3 + m3) * Kb;
      float acc = 0.f;
      for (int p = p0; p < p1; ++p) {
        const DevPath& q = d.path[p];
        const float* t = theta + q.theta_off + u;
        const float* ap = a + q.koff;
        for (int k = 0; k < d.R; ++k) acc = fmaf(t[size_t(k) * c], ap[size_t(k) * c], acc);
      }
      o[m3] = mode ? o[m3] + acc : acc;
    }
  }
}

__global__ void __launch_bounds__(kTX* kTY) k_cw_adjoint(const __grid_constant__ DevPlan d, int i3, int r0, int nc,
                                                         const float* __restrict__ g,
                                                         const float* __restrict__ theta, float* __restrict__ G) {
  const int c = d.out_mul[i3], n3 = 2 * d.out_l[i3] + 1, Kb = d.Kb[i3];
  const int j = blockIdx.y * kTX + threadIdx.x;
  if (j >= Kb) return;
  int k = 0, u = 0;
  const int p = cw_column(d, true, i3, j, &k, &u);
  if (p < 0) return;
  const float t = theta[d.path[p].theta_off + size_t(k) * c + u];
  float* Gb = G + size_t(nc) * d.a_pref[i3] + j;
  for (int n = blockIdx.x * kTY + threadIdx.y; n < nc; n += gridDim.x * kTY) {
    const float* gr = g + size_t(r0 + n) * d.dim_out + d.out_off[i3] + u * n3;
    for (int m3 = 0; m3 < n3; ++m3) Gb[(size_t(n) * n3 + m3) * Kb] = t * gr[m3];
  }
}

__global__ void __launch_bounds__(kTX* kTY) k_cw_dx(const __grid_constant__ DevPlan d, int i1, int s0, int nc,
                                                    const float* __restrict__ B, const float* __restrict__ theta,
                                                    float* __restrict__ dx) {
  const int c = d.in_mul[i1], n1 = 2 * d.in_l[i1] + 1, Kx = d.Kx[i1];
  const int u = blockIdx.y * kTX + threadIdx.x;
  if (u >= c) return;
  const float* Bb = B + size_t(nc) * d.b_pref[i1] + u;
  for (int n = blockIdx.x * kTY + threadIdx.y; n < nc; n += gridDim.x * kTY) {
    float* o = dx + size_t(s0 + n) * d.dim_in + d.in_off[i1] + u * n1;
    for (int m1 = 0; m1 < n1; ++m1) {
      const float* b = Bb + (size_t(n) * n1 + m1) * Kx;
      float acc = 0.f;
      for (int p = 0; p < d.P; ++p) {  // paths of one input block are not contiguous
        const DevPath& q = d.path[p];
        if (q.i1 != i1) continue;
        const float* t = theta + q.theta_off + u;
        const float* bp = b + q.kxoff;
        for (int k = 0; k < d.R; ++k) acc = fmaf(t[size_t(k) * c], bp[size_t(k) * c], acc);
      }
      o[m1] += acc;
    }
  }
}

// One Theta entry per column of the sender state; the y-rows of a block add
// their partial sums in shared memory, then one atomic add per column.
__global__ void __launch_bounds__(kTX* kTY) k_cw_dtheta(const __grid_constant__ DevPlan d, int i1, int s0, int nc,
                                                        const float* __restrict__ xa, const float* __restrict__ Ba,
                                                        const float* __restrict__ xb, const float* __restrict__ Bb,
                                                        float* __restrict__ dtheta) {
  __shared__ float red[kTY][kTX];
  const int c = d.in_mul[i1], n1 = 2 * d.in_l[i1] + 1, Kx = d.Kx[i1];
  const int j = blockIdx.y * kTX + threadIdx.x;
  int k = 0, u = 0;
  const int p = j < Kx ? cw_column(d, false, i1, j, &k, &u) : -1;
  float acc = 0.f;
  if (p >= 0) {
    const size_t boff = size_t(nc) * d.b_pref[i1] + j;
    for (int n = blockIdx.x * kTY + threadIdx.y; n < nc; n += gridDim.x * kTY) {
      const size_t xo = size_t(s0 + n) * d.dim_in + d.in_off[i1] + u * n1;
      const size_t bo = boff + size_t(n) * n1 * Kx;
      for (int m1 = 0; m1 < n1; ++m1) {
        if (xa) acc = fmaf(xa[xo + m1], Ba[bo + size_t(m1) * Kx], acc);
        if (xb) acc = fmaf(xb[xo + m1], Bb[bo + size_t(m1) * Kx], acc);
      }
    }
  }
  red[threadIdx.y][threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.y == 0 && p >= 0) {
    float s = 0.f;
#pragma unroll
    for (int y = 0; y < kTY; ++y) s += red[y][threadIdx.x];
    atomicAdd(dtheta + d.path[p].theta_off + size_t(k) * c + u, s);
  }
}

}  // namespace

cudaError_t cw_forward(const DevPlan& d, int r0, int nc, const float* A, const float* theta, float* out, int mode,
                       cudaStream_t st) {
  for (int i3 = 0; i3 < d.n_out; ++i3) {
    if (nc <= 0 || d.out_mul[i3] <= 0) continue;
    if (d.Kb[i3] == 0) {  // no path reaches this block: its output is zero
      if (mode == 0) {
        const size_t w = size_t(d.out_mul[i3]) * (2 * d.out_l[i3] + 1) * 4;
        cudaError_t e = cudaMemset2DAsync(out + size_t(r0) * d.dim_out + d.out_off[i3], size_t(d.dim_out) * 4, 0, w,
                                          size_t(nc), st);
        if (e) return e;
      }
      continue;
    }
    k_cw_forward<<<cw_grid(nc, d.out_mul[i3]), dim3(kTX, kTY), 0, st>>>(d, i3, r0, nc, A, theta, out, mode);
    cudaError_t e = cudaGetLastError();
    if (e) return e;
  }
  return cudaSuccess;
}

cudaError_t cw_adjoint(const DevPlan& d, int r0, int nc, const float* g, const float* theta, float* G,
                       cudaStream_t st) {
  for (int i3 = 0; i3 < d.n_out; ++i3) {
    if (nc <= 0 || d.Kb[i3] == 0) continue;
    k_cw_adjoint<<<cw_grid(nc, d.Kb[i3]), dim3(kTX, kTY), 0, st>>>(d, i3, r0, nc, g, theta, G);
    cudaError_t e = cudaGetLastError();
    if (e) return e;
  }
  return cudaSuccess;
}

cudaError_t cw_dx(const DevPlan& d, int s0, int nc, const float* B, const float* theta, float* dx, cudaStream_t st) {
  for (int i1 = 0; i1 < d.n_in; ++i1) {
    if (nc <= 0 || d.Kx[i1] == 0) continue;
    k_cw_dx<<<cw_grid(nc, d.in_mul[i1]), dim3(kTX, kTY), 0, st>>>(d, i1, s0, nc, B, theta, dx);
    cudaError_t e = cudaGetLastError();
    if (e) return e;
  }
  return cudaSuccess;
}

cudaError_t cw_dtheta(const DevPlan& d, int s0, int nc, const float* xa, const float* Ba, const float* xb,
                      const float* Bb, float* dtheta, cudaStream_t st) {
  if (!(xa && Ba) && !(xb && Bb)) return cudaSuccess;
  if (!(xa && Ba)) xa = Ba = nullptr;
  if (!(xb && Bb)) xb = Bb = nullptr;
  for (int i1 = 0; i1 < d.n_in; ++i1) {
    if (nc <= 0 || d.Kx[i1] == 0) continue;
    k_cw_dtheta<<<cw_grid(nc, d.Kx[i1]), dim3(kTX, kTY), 0, st>>>(d, i1, s0, nc, xa, Ba, xb, Bb, dtheta);
    cudaError_t e = cudaGetLastError();
    if (e) return e;
  }
  return cudaSuccess;
}

// launches issued by each entry point (for the caller's launch count)
int cw_launches_out(const DevPlan& d) {
  int n = 0;
  for (int i3 = 0; i3 < d.n_out; ++i3) n += d.Kb[i3] > 0;
  return n;
}
int cw_launches_in(const DevPlan& d) {
  int n = 0;
  for (int i1 = 0; i1 < d.n_in; ++i1) n += d.Kx[i1] > 0;
  return n;
}

}  // namespace tpc
