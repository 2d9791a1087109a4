// Node-level contractions of the channel-wise operator family (see channelwise.h).
//
// Two forms of each map:
//   * four channels per thread (every multiplicity a multiple of 4, Theta
//     16-byte aligned): one thread per (node, group of 4 channels or state
//     columns), rows of the block unrolled, state moved as float4 with
//     streaming loads / stores;
//   * one channel per thread otherwise: 32 x 8 thread blocks, x over 32
//     consecutive channels (or state columns), y over nodes, grid-strided,
//     about eight blocks per SM.
// Either way a warp reads or writes each state row as whole 128-byte lines.
// Theta is a few KB and stays in L1.  The Theta gradient reduces the node rows
// of a block in shared memory and adds one partial per Theta entry and block.
#include <cuda_runtime.h>

#include <stdint.h>

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

// ---- four channels per thread ---------------------------------------------
// When every multiplicity is a multiple of 4 (and Theta is 16-byte aligned),
// four consecutive channels share one radial index and path, so each thread
// moves whole float4 rows: A / B are streamed with 16-byte loads, G written
// with 16-byte stores.  N = 2l + 1 rows of the block are unrolled, so N
// independent 16-byte loads are in flight per (path, k) step.
constexpr int kT4 = 256;

__device__ __forceinline__ void fma4(float4& a, const float4& t, const float4& v) {
  a.x = fmaf(t.x, v.x, a.x);
  a.y = fmaf(t.y, v.y, a.y);
  a.z = fmaf(t.z, v.z, a.z);
  a.w = fmaf(t.w, v.w, a.w);
}
__device__ __forceinline__ float comp(const float4& v, int i) { return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w; }

// sum over the paths of one block (receiver: paths into i3; sender: paths from i1)
// of sum_k Theta[p][k][u..u+3] * S[row m, off_p + k c + u..u+3]
template <int N, bool RECV>
__device__ __forceinline__ void cw_sum4(const DevPlan& d, int blk, const float* __restrict__ S, int ld, int c, int u,
                                        const float* __restrict__ theta, float4 (&acc)[N]) {
  for (int p = 0; p < d.P; ++p) {
    const DevPath& q = d.path[p];
    if ((RECV ? q.i3 : q.i1) != blk) continue;
    const float* t = theta + q.theta_off + u;
    const float* sp = S + (RECV ? q.koff : q.kxoff) + u;
#pragma unroll 2
    for (int k = 0; k < d.R; ++k) {
      const float4 tk = __ldg(reinterpret_cast<const float4*>(t + size_t(k) * c));
#pragma unroll
      for (int m = 0; m < N; ++m)
        fma4(acc[m], tk, __ldcs(reinterpret_cast<const float4*>(sp + size_t(m) * ld + size_t(k) * c)));
    }
  }
}

// forward (RECV: A -> out) and dx (!RECV: B -> dx, accumulated)
template <int N, bool RECV>
__global__ void __launch_bounds__(kT4) k_cw_mix4(const __grid_constant__ DevPlan d, int blk, int r0, int nc,
                                                 const float* __restrict__ S, const float* __restrict__ theta,
                                                 float* __restrict__ out, int mode) {
  const int c = RECV ? d.out_mul[blk] : d.in_mul[blk];
  const int ld = RECV ? d.Kb[blk] : d.Kx[blk];
  const int cg = c >> 2;
  const int64_t idx = int64_t(blockIdx.x) * kT4 + threadIdx.x;
  if (idx >= int64_t(nc) * cg) return;
  const int n = int(idx / cg), u = int(idx - int64_t(n) * cg) * 4;
  const float* Sn = S + size_t(nc) * (RECV ? d.a_pref[blk] : d.b_pref[blk]) + size_t(n) * N * ld;
  float4 acc[N];
#pragma unroll
  for (int m = 0; m < N; ++m) acc[m] = make_float4(0.f, 0.f, 0.f, 0.f);
  cw_sum4<N, RECV>(d, blk, Sn, ld, c, u, theta, acc);
  const int dim = RECV ? d.dim_out : d.dim_in, off = RECV ? d.out_off[blk] : d.in_off[blk];
  float* o = out + size_t(r0 + n) * dim + off + u * N;  // channels u..u+3: 4N consecutive floats
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int m = 0; m < N; ++m) o[i * N + m] = (mode ? o[i * N + m] : 0.f) + comp(acc[m], i);
}

// G[(n, m), j..j+3] = Theta[p][k][u..u+3] * g[r0 + n, i3, u..u+3, m]
template <int N>
__global__ void __launch_bounds__(kT4) k_cw_adjoint4(const __grid_constant__ DevPlan d, int i3, int r0, int nc,
                                                     const float* __restrict__ g, const float* __restrict__ theta,
                                                     float* __restrict__ G) {
  const int Kb = d.Kb[i3], jg = Kb >> 2, c = d.out_mul[i3];
  const int64_t idx = int64_t(blockIdx.x) * kT4 + threadIdx.x;
  if (idx >= int64_t(nc) * jg) return;
  const int n = int(idx / jg), j = int(idx - int64_t(n) * jg) * 4;
  int k = 0, u = 0;
  const int p = cw_column(d, true, i3, j, &k, &u);
  if (p < 0) return;
  const float4 t = __ldg(reinterpret_cast<const float4*>(theta + d.path[p].theta_off + size_t(k) * c + u));
  const float* gr = g + size_t(r0 + n) * d.dim_out + d.out_off[i3] + u * N;
  float* Gn = G + size_t(nc) * d.a_pref[i3] + size_t(n) * N * Kb + j;
#pragma unroll
  for (int m = 0; m < N; ++m)
    __stcs(reinterpret_cast<float4*>(Gn + size_t(m) * Kb),
           make_float4(t.x * gr[m], t.y * gr[N + m], t.z * gr[2 * N + m], t.w * gr[3 * N + m]));
}

// dTheta over four columns per thread; y-rows of a block reduce in shared memory
template <int N>
__global__ void __launch_bounds__(kTX* kTY) k_cw_dtheta4(const __grid_constant__ DevPlan d, int i1, int s0, int nc,
                                                         const float* __restrict__ xa, const float* __restrict__ Ba,
                                                         const float* __restrict__ xb, const float* __restrict__ Bb,
                                                         float* __restrict__ dtheta) {
  __shared__ float4 red[kTY][kTX];
  const int Kx = d.Kx[i1], c = d.in_mul[i1];
  const int j = (blockIdx.y * kTX + threadIdx.x) * 4;
  int k = 0, u = 0;
  const int p = j < Kx ? cw_column(d, false, i1, j, &k, &u) : -1;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (p >= 0) {
    const size_t boff = size_t(nc) * d.b_pref[i1] + j;
    for (int n = blockIdx.x * kTY + threadIdx.y; n < nc; n += gridDim.x * kTY) {
      const size_t xo = size_t(s0 + n) * d.dim_in + d.in_off[i1] + u * N;
      const size_t bo = boff + size_t(n) * N * Kx;
#pragma unroll
      for (int m = 0; m < N; ++m) {
        if (xa) {
          const float4 b = __ldcs(reinterpret_cast<const float4*>(Ba + bo + size_t(m) * Kx));
          fma4(acc, make_float4(xa[xo + m], xa[xo + N + m], xa[xo + 2 * N + m], xa[xo + 3 * N + m]), b);
        }
        if (xb) {
          const float4 b = __ldcs(reinterpret_cast<const float4*>(Bb + bo + size_t(m) * Kx));
          fma4(acc, make_float4(xb[xo + m], xb[xo + N + m], xb[xo + 2 * N + m], xb[xo + 3 * N + m]), b);
        }
      }
    }
  }
  red[threadIdx.y][threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.y == 0 && p >= 0) {
    float4 s = red[0][threadIdx.x];
#pragma unroll
    for (int y = 1; y < kTY; ++y) {
      const float4 v = red[y][threadIdx.x];
      s.x += v.x;
      s.y += v.y;
      s.z += v.z;
      s.w += v.w;
    }
    float* dt = dtheta + d.path[p].theta_off + size_t(k) * c + u;
    atomicAdd(dt, s.x);
    atomicAdd(dt + 1, s.y);
    atomicAdd(dt + 2, s.z);
    atomicAdd(dt + 3, s.w);
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// the float4 kernels apply: multiplicities (and so every state column offset) multiples of 4
bool four_channels(const DevPlan& d) {
  for (int i = 0; i < d.n_in; ++i)
    if (d.in_mul[i] % 4) return false;
  for (int i = 0; i < d.n_out; ++i)
    if (d.out_mul[i] % 4 || d.Kb[i] % 4) return false;
  return true;
}

unsigned blocks_for(int64_t threads) { return unsigned((threads + kT4 - 1) / kT4); }

template <bool RECV>
cudaError_t launch_mix4(const DevPlan& d, int blk, int r0, int nc, const float* S, const float* theta, float* out,
                        int mode, cudaStream_t st) {
  const int c = RECV ? d.out_mul[blk] : d.in_mul[blk];
  const int l = RECV ? d.out_l[blk] : d.in_l[blk];
  const unsigned nb = blocks_for(int64_t(nc) * (c / 4));
  switch (2 * l + 1) {
    case 1: k_cw_mix4<1, RECV><<<nb, kT4, 0, st>>>(d, blk, r0, nc, S, theta, out, mode); break;
    case 3: k_cw_mix4<3, RECV><<<nb, kT4, 0, st>>>(d, blk, r0, nc, S, theta, out, mode); break;
    case 5: k_cw_mix4<5, RECV><<<nb, kT4, 0, st>>>(d, blk, r0, nc, S, theta, out, mode); break;
    default: k_cw_mix4<7, RECV><<<nb, kT4, 0, st>>>(d, blk, r0, nc, S, theta, out, mode); break;
  }
  return cudaGetLastError();
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
    cudaError_t e;
    if (four_channels(d) && aligned16(theta)) {
      e = launch_mix4<true>(d, i3, r0, nc, A, theta, out, mode, st);
    } else {
      k_cw_forward<<<cw_grid(nc, d.out_mul[i3]), dim3(kTX, kTY), 0, st>>>(d, i3, r0, nc, A, theta, out, mode);
      e = cudaGetLastError();
    }
    if (e) return e;
  }
  return cudaSuccess;
}

cudaError_t cw_adjoint(const DevPlan& d, int r0, int nc, const float* g, const float* theta, float* G,
                       cudaStream_t st) {
  for (int i3 = 0; i3 < d.n_out; ++i3) {
    if (nc <= 0 || d.Kb[i3] == 0) continue;
    if (four_channels(d) && aligned16(theta)) {
      const unsigned nb = blocks_for(int64_t(nc) * (d.Kb[i3] / 4));
      switch (2 * d.out_l[i3] + 1) {
        case 1: k_cw_adjoint4<1><<<nb, kT4, 0, st>>>(d, i3, r0, nc, g, theta, G); break;
        case 3: k_cw_adjoint4<3><<<nb, kT4, 0, st>>>(d, i3, r0, nc, g, theta, G); break;
        case 5: k_cw_adjoint4<5><<<nb, kT4, 0, st>>>(d, i3, r0, nc, g, theta, G); break;
        default: k_cw_adjoint4<7><<<nb, kT4, 0, st>>>(d, i3, r0, nc, g, theta, G); break;
      }
    } else {
      k_cw_adjoint<<<cw_grid(nc, d.Kb[i3]), dim3(kTX, kTY), 0, st>>>(d, i3, r0, nc, g, theta, G);
    }
    cudaError_t e = cudaGetLastError();
    if (e) return e;
  }
  return cudaSuccess;
}

cudaError_t cw_dx(const DevPlan& d, int s0, int nc, const float* B, const float* theta, float* dx, cudaStream_t st) {
  for (int i1 = 0; i1 < d.n_in; ++i1) {
    if (nc <= 0 || d.Kx[i1] == 0) continue;
    cudaError_t e;
    if (four_channels(d) && aligned16(theta)) {
      e = launch_mix4<false>(d, i1, s0, nc, B, theta, dx, 1, st);
    } else {
      k_cw_dx<<<cw_grid(nc, d.in_mul[i1]), dim3(kTX, kTY), 0, st>>>(d, i1, s0, nc, B, theta, dx);
      e = cudaGetLastError();
    }
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
    if (four_channels(d)) {
      const dim3 grid = cw_grid(nc, d.Kx[i1] / 4);
      switch (2 * d.in_l[i1] + 1) {
        case 1: k_cw_dtheta4<1><<<grid, dim3(kTX, kTY), 0, st>>>(d, i1, s0, nc, xa, Ba, xb, Bb, dtheta); break;
        case 3: k_cw_dtheta4<3><<<grid, dim3(kTX, kTY), 0, st>>>(d, i1, s0, nc, xa, Ba, xb, Bb, dtheta); break;
        case 5: k_cw_dtheta4<5><<<grid, dim3(kTX, kTY), 0, st>>>(d, i1, s0, nc, xa, Ba, xb, Bb, dtheta); break;
        default: k_cw_dtheta4<7><<<grid, dim3(kTX, kTY), 0, st>>>(d, i1, s0, nc, xa, Ba, xb, Bb, dtheta); break;
      }
    } else {
      k_cw_dtheta<<<cw_grid(nc, d.Kx[i1]), dim3(kTX, kTY), 0, st>>>(d, i1, s0, nc, xa, Ba, xb, Bb, dtheta);
    }
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
