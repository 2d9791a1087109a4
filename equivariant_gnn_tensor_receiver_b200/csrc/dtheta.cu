// Theta gradient of the streaming schedule: for every path p (input block i1),
//
//     dTheta[p][k][u][w] += sum_{s in chunk} sum_m1 x[s, u, m1] * B[s, k, w, m1]
//
// (and a second pair xb, Bb in the same pass for the double backward).  As a
// GEMM per path: M = c_in (u), N = R * c_out (the contiguous (k, w) columns of
// the path's B block), K = (node, m1) over the chunk.  K is long (nodes x
// (2 l1 + 1)) and M x N small, so the K range is split over CTAs that add their
// partial tiles with red.global.add into the zeroed gradient.  A CTA owns a
// 64 (u) x 256 (k, w) tile; stages of about 40 K rows are gathered with cp.async
// into a double buffer (x transposed to [row][u] on the way in), and each
// thread keeps an 8 x 8 accumulator tile fed by four 16-byte shared reads per
// 32 paired FMAs (the u octet is a warp-wide broadcast).
#include <cuda_runtime.h>

#include <algorithm>

#include "async_copy.cuh"
#include "dtheta.h"

namespace tpc {
namespace {

constexpr int kTU = 64;    // u per CTA tile
constexpr int kTN = 256;   // (k, w) columns per CTA tile
constexpr int kThreads = 256;

template <int N1>
struct DtCfg {
  static constexpr int TS = 40 / N1;             // nodes per stage
  static constexpr int ROWS = TS * N1;           // K rows per stage
  static constexpr int XS = ROWS * kTU;          // transposed x: [row][u]
  static constexpr int STAGE = XS + ROWS * kTN;  // + B: [row][n]
};
constexpr int cmax(int a, int b) { return a > b ? a : b; }
constexpr int kStageMax =  // floats of one stage buffer, largest over 2 l1 + 1
    cmax(cmax(DtCfg<1>::STAGE, DtCfg<3>::STAGE), cmax(DtCfg<5>::STAGE, DtCfg<7>::STAGE));
constexpr int smem_bytes() { return 2 * kStageMax * 4; }

// gather ns nodes of one (x, B) pair into a stage buffer
template <int N1>
__device__ __forceinline__ void dt_stage(float* st, int ns, const float* __restrict__ x, size_t xrow0, int dim_in,
                                         int cu, const float* __restrict__ B, size_t brow0, int ldb, int cn,
                                         bool v4) {
  using C = DtCfg<N1>;
  float* sX = st;
  float* sB = st + C::XS;
  constexpr int XW = kTU * N1;
  for (int t = threadIdx.x; t < ns * XW; t += kThreads) {
    const int j = t / XW, o = t - j * XW;  // o = u * N1 + m1
    const int u = o / N1, m1 = o - u * N1;
    float* dst = sX + (j * N1 + m1) * kTU + u;
    if (u < cu) ac_copy4(dst, x + xrow0 + size_t(j) * dim_in + o);
    else *dst = 0.f;
  }
  const int rows = ns * N1;
  if (v4) {
    for (int t = threadIdx.x; t < rows * (kTN / 4); t += kThreads) {
      const int r = t / (kTN / 4), c = 4 * (t - r * (kTN / 4));
      float* dst = sB + r * kTN + c;
      if (c < cn) ac_copy16(dst, B + brow0 + size_t(r) * ldb + c);
      else sts4(dst, 0.f, 0.f, 0.f, 0.f);
    }
  } else {
    for (int t = threadIdx.x; t < rows * kTN; t += kThreads) {
      const int r = t / kTN, c = t - r * kTN;
      float* dst = sB + r * kTN + c;
      if (c < cn) ac_copy4(dst, B + brow0 + size_t(r) * ldb + c);
      else *dst = 0.f;
    }
  }
}

template <int N1>
__device__ __forceinline__ void tile(const DevPlan& pl, const DevPath& q, int u0, int n0, int sb, int se, int s0,
                                     int nc, const float* __restrict__ xa, const float* __restrict__ Ba,
                                     const float* __restrict__ xb, const float* __restrict__ Bb,
                                     float* __restrict__ dtheta, float* sm) {
  using C = DtCfg<N1>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cu = min(kTU, q.c_in - u0);
  const int cn = min(kTN, pl.R * q.c_out - n0);
  const int ldb = pl.Kx[q.i1];
  const float* xs[2] = {xa, xb};
  const float* Bs[2] = {Ba, Bb};
  const int nst1 = (se - sb + C::TS - 1) / C::TS;  // stages per pair
  const int npair = (xa && Ba ? 1 : 0) + (xb && Bb ? 1 : 0);
  const int first = (xa && Ba) ? 0 : 1;
  const int nst = npair * nst1;
  auto stage = [&](int it) {
    const int pair = first + it / nst1, sc = sb + (it % nst1) * C::TS;
    const int ns = min(C::TS, se - sc);
    const float* x = xs[pair];
    const float* B = Bs[pair] + size_t(nc) * pl.b_pref[q.i1] + q.kxoff + n0;
    const bool v4 = ((reinterpret_cast<uintptr_t>(B) | size_t(ldb) * 4) & 15) == 0;
    dt_stage<N1>(sm + (it & 1) * kStageMax, ns, x, size_t(s0 + sc) * pl.dim_in + q.in_off + size_t(u0) * N1,
                 pl.dim_in, cu, B, size_t(sc) * N1 * ldb, ldb, cn, v4);
  };
  float2 acc[8][4];  // column pairs (2cp, 2cp+1) of the thread's 8 columns
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[i][c] = make_float2(0.f, 0.f);
  if (nst > 0) stage(0);
  ac_commit();
  for (int it = 0; it < nst; ++it) {
    if (it + 1 < nst) stage(it + 1);
    ac_commit();
    ac_wait<1>();
    __syncthreads();
    const float* sX = sm + (it & 1) * kStageMax;
    const float* sB = sX + C::XS;
    const int sc = sb + (it % nst1) * C::TS;
    const int rows = min(C::TS, se - sc) * N1;
    for (int r = 0; r < rows; ++r) {
      float a[8];
      float2 b[4];
      lds_vec<8>(sX + r * kTU + 8 * warp, a);
      lds_f2<2>(sB + r * kTN + 4 * lane, b);
      lds_f2<2>(sB + r * kTN + 128 + 4 * lane, b + 2);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 ai = make_float2(a[i], a[i]);
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][c] = __ffma2_rn(ai, b[c], acc[i][c]);
      }
    }
    __syncthreads();
  }
  // dTheta[p][k][u][w], column n = k * c_out + w
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int u = 8 * warp + i;
    if (u >= cu) continue;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int n = c < 4 ? 4 * lane + c : 128 + 4 * lane + c - 4;
      if (n >= cn) continue;
      const int ng = n0 + n, k = ng / q.c_out, w = ng - k * q.c_out;
      const float v = (c & 1) ? acc[i][c >> 1].y : acc[i][c >> 1].x;
      atomicAdd(dtheta + q.theta_off + (size_t(k) * q.c_in + u0 + u) * q.c_out + w, v);
    }
  }
}

// grid.x: tiles (p, u tile, n tile) over the plan's largest extents, grid.y: K splits.
// A split holds about rows_per_split K rows: nodes x (2 l1 + 1) of its path, so the
// CTAs of every path carry the same work and one wave ends together.
__global__ void __launch_bounds__(kThreads, 2)
    k_dtheta(const __grid_constant__ DevPlan pl, int s0, int nc, int ut, int nt, int rows_per_split,
             const float* __restrict__ xa, const float* __restrict__ Ba, const float* __restrict__ xb,
             const float* __restrict__ Bb, float* __restrict__ dtheta) {
  extern __shared__ __align__(16) float sm[];
  const int t = blockIdx.x;
  const int p = t / (ut * nt), r = t - p * (ut * nt);
  const DevPath& q = pl.path[p];
  const int u0 = (r / nt) * kTU, n0 = (r % nt) * kTN;
  if (u0 >= q.c_in || n0 >= pl.R * q.c_out) return;
  const int n1 = 2 * q.l1 + 1;
  const int nodes_per_split = max(1, (rows_per_split + n1 - 1) / n1);
  if (int64_t(blockIdx.y) * nodes_per_split >= nc) return;
  const int sb = blockIdx.y * nodes_per_split, se = min(nc, sb + nodes_per_split);
  switch (q.l1) {
    case 0: tile<1>(pl, q, u0, n0, sb, se, s0, nc, xa, Ba, xb, Bb, dtheta, sm); break;
    case 1: tile<3>(pl, q, u0, n0, sb, se, s0, nc, xa, Ba, xb, Bb, dtheta, sm); break;
    case 2: tile<5>(pl, q, u0, n0, sb, se, s0, nc, xa, Ba, xb, Bb, dtheta, sm); break;
    default: tile<7>(pl, q, u0, n0, sb, se, s0, nc, xa, Ba, xb, Bb, dtheta, sm); break;
  }
}

}  // namespace

cudaError_t dtheta_smem_init() {
  return cudaFuncSetAttribute(k_dtheta, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes());
}

cudaError_t dtheta_accumulate(const DevPlan& d, int s0, int nc, const float* xa, const float* Ba, const float* xb,
                              const float* Bb, float* dtheta, cudaStream_t st) {
  if (nc <= 0 || d.P <= 0 || (!(xa && Ba) && !(xb && Bb))) return cudaSuccess;
  const int ut = (d.max_c_in + kTU - 1) / kTU;
  const int nt = (d.R * d.max_c_out + kTN - 1) / kTN;
  const int tiles = d.P * ut * nt;
  // One wave of two CTAs per SM with equal K rows per CTA: the rows of all
  // (non-empty) tiles over the slots, grown until the split count fits.
  const int slots = 2 * 148;
  int64_t rows = 0;
  int n1max = 1;
  for (int p = 0; p < d.P; ++p) {
    const DevPath& q = d.path[p];
    const int64_t tp = int64_t((q.c_in + kTU - 1) / kTU) * ((d.R * q.c_out + kTN - 1) / kTN);
    rows += tp * nc * (2 * q.l1 + 1);
    n1max = std::max(n1max, 2 * int(q.l1) + 1);
  }
  int64_t per = std::max<int64_t>(16, (rows + slots - 1) / slots);
  auto ctas = [&](int64_t rp, int64_t* ymax) {
    int64_t n = 0;
    *ymax = 1;
    for (int p = 0; p < d.P; ++p) {
      const DevPath& q = d.path[p];
      const int64_t tp = int64_t((q.c_in + kTU - 1) / kTU) * ((d.R * q.c_out + kTN - 1) / kTN);
      const int64_t n1 = 2 * q.l1 + 1, nps = std::max<int64_t>(1, (rp + n1 - 1) / n1);
      const int64_t y = (nc + nps - 1) / nps;
      n += tp * y;
      *ymax = std::max(*ymax, y);
    }
    return n;
  };
  int64_t ymax = 1;
  while (ctas(per, &ymax) > slots && per < int64_t(nc) * n1max) per += per / 16 + 1;
  ctas(per, &ymax);
  const dim3 grid(static_cast<unsigned>(tiles), static_cast<unsigned>(ymax));
  k_dtheta<<<grid, kThreads, smem_bytes(), st>>>(d, s0, nc, ut, nt, int(std::min<int64_t>(per, 1 << 30)), xa, Ba, xb,
                                                 Bb, dtheta);
  return cudaGetLastError();
}

}  // namespace tpc
