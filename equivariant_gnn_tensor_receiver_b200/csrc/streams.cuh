// Edge-stream kernels of the streaming schedule ("Sobek", arXiv 2607.18074,
// abstract: edge-local products are consumed directly into bounded node-side
// state; nothing edge-sized is materialised).
//
// Work decomposition: one warp per (node, path, channel tile of 32); lane =
// channel.  A lane keeps the node-side state of its (path, channel) in registers
// for the node's whole edge segment.  Per batch of kEdgeBatch edges the warp
// evaluates, with lane = edge, the edge geometry (spherical harmonics of degree
// l2, radial basis) and the edge's coupling matrix
//     M_e[m1][m3] = sum_m2 C_p[m1, m2, m3] Y_{l2 m2}(v_e)
// (structural zeros removed at compile time) into warp-private shared memory;
// the channel loop then runs FFMA on registers with broadcast shared reads.
//
//  k_fwd_path    receiver-sorted:  A[r, k, p, u, m3] = sum_e b_ek sum_m1 M_e[m1][m3] x[s_e, u, m1]
//  k_send_path   sender-sorted:    B[s, k, p, w, m1] = sum_e b_ek sum_m3 M_e[m1][m3] g[r_e, w, m3]
//  k_radj_stream receiver-sorted with G[r] = Theta^T g[r] resident in registers:
//                db_ek  = sum_{p,u,m3} G[r, k, p, u, m3] T_e[p, u, m3]
//                dY_e   = sum_p sum C_p x[s_e] (sum_k b_ek G[r, k, p])
//                dvec_e = J_Y(v_e)^T dY_e + J_b(v_e)^T db_e       (dual numbers)
//
// A / G column layout per output block i3: row (node, m3), column koff(p) + k*C_in + u.
// B column layout per input block i1:      row (node, m1), column kxoff(p) + k*C_out + w.
#pragma once

#include "common.cuh"

namespace tpc {

constexpr int kWarpsPerBlock = 4;

// ---- per-batch edge preparation (lane = edge) ----------------------------
template <int L1, int L2, int L3, int RM>
__device__ __forceinline__ void prep_edge(const DevPlan& pl, float vx, float vy, float vz, float* sM,
                                          float* sB) {
  using TR = Tri<L1, L2, L3>;
  constexpr int NMZ = TR::NMZ;
  float nx, ny, nz, r;
  unit(vx, vy, vz, nx, ny, nz, r);
  float Y[TR::N2];
  sh_degree<L2>(nx, ny, nz, Y);
  float b[RM];
  radial_basis<RM>(pl, r, b);
  float* Mrow = sM + lane_id() * NMZ;
  sfor<TR::N1>([&](auto I1) {
    sfor<TR::N3>([&](auto I3) {
      constexpr int i1 = decltype(I1)::value, i3 = decltype(I3)::value;
      if constexpr (TR::tab.m[i1][i3]) {
        float s = 0.f;
        sfor<TR::N2>([&](auto I2) {
          constexpr int i2 = decltype(I2)::value;
          if constexpr (TR::tab.cg[i1][i2][i3]) s = fmaf(TR::template cg<i1, i2, i3>(), Y[i2], s);
        });
        constexpr int mi = TR::tab.mi[i1][i3];
        Mrow[mi] = s;
      }
    });
  });
#pragma unroll
  for (int k = 0; k < RM; ++k) sB[lane_id() * RM + k] = b[k];
}

// compact coupling matrix of one degree-L2 vector into Mrow
template <int L1, int L2, int L3>
__device__ __forceinline__ void coupling_row(const float* Y, float* Mrow) {
  using TR = Tri<L1, L2, L3>;
  sfor<TR::N1>([&](auto I1) {
    sfor<TR::N3>([&](auto I3) {
      constexpr int i1 = decltype(I1)::value, i3 = decltype(I3)::value;
      if constexpr (TR::tab.m[i1][i3]) {
        float s = 0.f;
        sfor<TR::N2>([&](auto I2) {
          constexpr int i2 = decltype(I2)::value;
          if constexpr (TR::tab.cg[i1][i2][i3]) s = fmaf(TR::template cg<i1, i2, i3>(), Y[i2], s);
        });
        constexpr int mi = TR::tab.mi[i1][i3];
        Mrow[mi] = s;
      }
    });
  });
}

// T[m3] = sum_m1 M[m1][m3] x[m1]
template <int L1, int L2, int L3>
__device__ __forceinline__ void apply_M(const float* __restrict__ Mj, const float* xv, float* T) {
  using TR = Tri<L1, L2, L3>;
#pragma unroll
  for (int i3 = 0; i3 < TR::N3; ++i3) T[i3] = 0.f;
  sfor<TR::N1>([&](auto I1) {
    sfor<TR::N3>([&](auto I3) {
      constexpr int i1 = decltype(I1)::value, i3 = decltype(I3)::value;
      if constexpr (TR::tab.m[i1][i3]) {
        constexpr int mi = TR::tab.mi[i1][i3];
        T[i3] = fmaf(Mj[mi], xv[i1], T[i3]);
      }
    });
  });
}

// U[m1] = sum_m3 M[m1][m3] y[m3]
template <int L1, int L2, int L3>
__device__ __forceinline__ void apply_Mt(const float* __restrict__ Mj, const float* yv, float* U) {
  using TR = Tri<L1, L2, L3>;
#pragma unroll
  for (int i1 = 0; i1 < TR::N1; ++i1) U[i1] = 0.f;
  sfor<TR::N1>([&](auto I1) {
    sfor<TR::N3>([&](auto I3) {
      constexpr int i1 = decltype(I1)::value, i3 = decltype(I3)::value;
      if constexpr (TR::tab.m[i1][i3]) {
        constexpr int mi = TR::tab.mi[i1][i3];
        U[i1] = fmaf(Mj[mi], yv[i3], U[i1]);
      }
    });
  });
}

// Paired forms for a coupling matrix and its derivative stored side by side,
// MM[mi] = (M[mi], Md[mi]): one paired FMA applies both.
// (T[m3], Td[m3]) = sum_m1 (M, Md)[m1][m3] x[m1]
template <int L1, int L2, int L3>
__device__ __forceinline__ void apply_M2(const float2* MM, const float* xv, float2* TT) {
  using TR = Tri<L1, L2, L3>;
#pragma unroll
  for (int i3 = 0; i3 < TR::N3; ++i3) TT[i3] = make_float2(0.f, 0.f);
  sfor<TR::N1>([&](auto I1) {
    sfor<TR::N3>([&](auto I3) {
      constexpr int i1 = decltype(I1)::value, i3 = decltype(I3)::value;
      if constexpr (TR::tab.m[i1][i3]) {
        constexpr int mi = TR::tab.mi[i1][i3];
        TT[i3] = __ffma2_rn(MM[mi], make_float2(xv[i1], xv[i1]), TT[i3]);
      }
    });
  });
}
// (U[m1], Ud[m1]) = sum_m3 (M, Md)[m1][m3] y[m3]
template <int L1, int L2, int L3>
__device__ __forceinline__ void apply_Mt2(const float2* MM, const float* yv, float2* UU) {
  using TR = Tri<L1, L2, L3>;
#pragma unroll
  for (int i1 = 0; i1 < TR::N1; ++i1) UU[i1] = make_float2(0.f, 0.f);
  sfor<TR::N1>([&](auto I1) {
    sfor<TR::N3>([&](auto I3) {
      constexpr int i1 = decltype(I1)::value, i3 = decltype(I3)::value;
      if constexpr (TR::tab.m[i1][i3]) {
        constexpr int mi = TR::tab.mi[i1][i3];
        UU[i1] = __ffma2_rn(MM[mi], make_float2(yv[i3], yv[i3]), UU[i1]);
      }
    });
  });
}
// T[m3] = sum_m1 M[m1][m3] x[m1] with M the first members of MM
template <int L1, int L2, int L3>
__device__ __forceinline__ void apply_M_first(const float2* MM, const float* xv, float* T) {
  using TR = Tri<L1, L2, L3>;
#pragma unroll
  for (int i3 = 0; i3 < TR::N3; ++i3) T[i3] = 0.f;
  sfor<TR::N1>([&](auto I1) {
    sfor<TR::N3>([&](auto I3) {
      constexpr int i1 = decltype(I1)::value, i3 = decltype(I3)::value;
      if constexpr (TR::tab.m[i1][i3]) {
        constexpr int mi = TR::tab.mi[i1][i3];
        T[i3] = fmaf(MM[mi].x, xv[i1], T[i3]);
      }
    });
  });
}

// out[m2] = sum_{m1,m3} C[m1,m2,m3] a[m1] c[m3]
template <int L1, int L2, int L3>
__device__ __forceinline__ void cg_contract_13(const float* a, const float* c, float* out) {
  using TR = Tri<L1, L2, L3>;
#pragma unroll
  for (int i2 = 0; i2 < TR::N2; ++i2) out[i2] = 0.f;
  sfor<TR::N1>([&](auto I1) {
    sfor<TR::N3>([&](auto I3) {
      constexpr int i1 = decltype(I1)::value, i3 = decltype(I3)::value;
      if constexpr (TR::tab.m[i1][i3]) {
        const float ac = a[i1] * c[i3];
        sfor<TR::N2>([&](auto I2) {
          constexpr int i2 = decltype(I2)::value;
          if constexpr (TR::tab.cg[i1][i2][i3]) out[i2] = fmaf(TR::template cg<i1, i2, i3>(), ac, out[i2]);
        });
      }
    });
  });
}

// ===========================================================================
// forward receiver stream, one path: grid (ceil(nc / 4), channel tiles), 4 warps
// ===========================================================================
template <int L1, int L2, int L3, int RM>
__global__ void __launch_bounds__(32 * kWarpsPerBlock)
    k_fwd_path(const __grid_constant__ DevPlan pl, int p, int r0, int nc, const int* __restrict__ rowptr,
               const int* __restrict__ col, const float* __restrict__ vec, const float* __restrict__ x,
               float* __restrict__ A) {
  using TR = Tri<L1, L2, L3>;
  constexpr int N1 = TR::N1, N3 = TR::N3, NMZ = TR::NMZ, EB = kEdgeBatch;
  constexpr int WS = EB * (NMZ + RM + 1);
  __shared__ float smem[kWarpsPerBlock * WS];
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const int rl = blockIdx.x * kWarpsPerBlock + warp;
  if (rl >= nc) return;
  const DevPath& pa = pl.path[p];
  float* sM = smem + warp * WS;
  float* sB = sM + EB * NMZ;
  int* sS = reinterpret_cast<int*>(sB + EB * RM);
  const int u = blockIdx.y * 32 + lane;
  const bool active = u < pa.c_in;
  float acc[RM][N3];
#pragma unroll
  for (int k = 0; k < RM; ++k)
#pragma unroll
    for (int i = 0; i < N3; ++i) acc[k][i] = 0.f;

  const int r = r0 + rl;
  const int e0 = rowptr[r], e1 = rowptr[r + 1];
  const float* xb = x + pa.in_off + size_t(active ? u : 0) * N1;
  for (int eb = e0; eb < e1; eb += EB) {
    const int nb = min(EB, e1 - eb);
    __syncwarp();
    if (lane < nb) {
      const int e = eb + lane;
      prep_edge<L1, L2, L3, RM>(pl, vec[3 * e], vec[3 * e + 1], vec[3 * e + 2], sM, sB);
      sS[lane] = col[e];
    }
    __syncwarp();
#pragma unroll 2
    for (int j = 0; j < nb; ++j) {
      const float* xp = xb + size_t(sS[j]) * pl.dim_in;
      float xv[N1];
#pragma unroll
      for (int i = 0; i < N1; ++i) xv[i] = active ? __ldg(xp + i) : 0.f;
      float T[N3];
      apply_M<L1, L2, L3>(sM + j * NMZ, xv, T);
#pragma unroll
      for (int k = 0; k < RM; ++k) {
        const float bk = sB[j * RM + k];
#pragma unroll
        for (int i = 0; i < N3; ++i) acc[k][i] = fmaf(bk, T[i], acc[k][i]);
      }
    }
  }
  if (!active) return;
  const int Kb = pl.Kb[pa.i3];
  float* Ablk = A + size_t(nc) * pl.a_pref[pa.i3];
#pragma unroll
  for (int k = 0; k < RM; ++k) {
    if (k >= pl.R) break;
#pragma unroll
    for (int i = 0; i < N3; ++i) Ablk[size_t(rl * N3 + i) * Kb + pa.koff + k * pa.c_in + u] = acc[k][i];
  }
}

// ===========================================================================
// backward sender stream, one path: B[s] = sum_{e in out(s)} b_e (x) M_e^T g[r_e]
// ===========================================================================
template <int L1, int L2, int L3, int RM>
__global__ void __launch_bounds__(32 * kWarpsPerBlock)
    k_send_path(const __grid_constant__ DevPlan pl, int p, int s0, int nc, const int* __restrict__ s_rowptr,
                const int* __restrict__ perm, const int* __restrict__ s_recv, const float* __restrict__ vec,
                const float* __restrict__ g, float* __restrict__ B) {
  using TR = Tri<L1, L2, L3>;
  constexpr int N1 = TR::N1, N3 = TR::N3, NMZ = TR::NMZ, EB = kEdgeBatch;
  constexpr int WS = EB * (NMZ + RM + 1);
  __shared__ float smem[kWarpsPerBlock * WS];
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const int sl = blockIdx.x * kWarpsPerBlock + warp;
  if (sl >= nc) return;
  const DevPath& pa = pl.path[p];
  float* sM = smem + warp * WS;
  float* sB = sM + EB * NMZ;
  int* sR = reinterpret_cast<int*>(sB + EB * RM);
  const int w = blockIdx.y * 32 + lane;
  const bool active = w < pa.c_out;
  float acc[RM][N1];
#pragma unroll
  for (int k = 0; k < RM; ++k)
#pragma unroll
    for (int i = 0; i < N1; ++i) acc[k][i] = 0.f;

  const int s = s0 + sl;
  const int j0 = s_rowptr[s], j1 = s_rowptr[s + 1];
  const float* gb = g + pa.out_off + size_t(active ? w : 0) * N3;
  for (int jb = j0; jb < j1; jb += EB) {
    const int nb = min(EB, j1 - jb);
    __syncwarp();
    if (lane < nb) {
      const int e = perm[jb + lane];
      prep_edge<L1, L2, L3, RM>(pl, vec[3 * e], vec[3 * e + 1], vec[3 * e + 2], sM, sB);
      sR[lane] = s_recv[jb + lane];
    }
    __syncwarp();
#pragma unroll 2
    for (int j = 0; j < nb; ++j) {
      const float* gp = gb + size_t(sR[j]) * pl.dim_out;
      float gv[N3];
#pragma unroll
      for (int i = 0; i < N3; ++i) gv[i] = active ? __ldg(gp + i) : 0.f;
      float U[N1];
      apply_Mt<L1, L2, L3>(sM + j * NMZ, gv, U);
#pragma unroll
      for (int k = 0; k < RM; ++k) {
        const float bk = sB[j * RM + k];
#pragma unroll
        for (int i = 0; i < N1; ++i) acc[k][i] = fmaf(bk, U[i], acc[k][i]);
      }
    }
  }
  if (!active) return;
  const int Kx = pl.Kx[pa.i1];
  float* Bblk = B + size_t(nc) * pl.b_pref[pa.i1];
#pragma unroll
  for (int k = 0; k < RM; ++k) {
    if (k >= pl.R) break;
#pragma unroll
    for (int i = 0; i < N1; ++i) Bblk[size_t(sl * N1 + i) * Kx + pa.kxoff + k * pa.c_out + w] = acc[k][i];
  }
}

// ===========================================================================
// backward receiver adjoint stream: per-edge dY, db -> dvec (all paths in a CTA)
// ===========================================================================
// One window of up to kEdgeBatch edges of receiver r for path p, all channel
// tiles.  Leaves this path's reduced (dY_l2 block, db) in sAcc[j][N2 + RM].
template <int L1, int L2, int L3, int RM>
__device__ __forceinline__ void radj_path(const DevPlan& pl, const DevPath& pa, int rl, int eb, int nb,
                                          const int* __restrict__ col, const float* __restrict__ vec,
                                          const float* __restrict__ x, const float* __restrict__ Gblk,
                                          float* sm) {
  using TR = Tri<L1, L2, L3>;
  constexpr int N1 = TR::N1, N2 = TR::N2, N3 = TR::N3, NMZ = TR::NMZ, EB = kEdgeBatch;
  float* sM = sm;
  float* sB = sM + EB * NMZ;
  int* sS = reinterpret_cast<int*>(sB + EB * RM);
  float* sAcc = reinterpret_cast<float*>(sS + EB);  // [EB][N2 + RM]
  const int lane = lane_id();
  __syncwarp();
  if (lane < nb) {
    const int e = eb + lane;
    prep_edge<L1, L2, L3, RM>(pl, vec[3 * e], vec[3 * e + 1], vec[3 * e + 2], sM, sB);
    sS[lane] = col[e];
  }
  for (int i = lane; i < EB * (N2 + RM); i += 32) sAcc[i] = 0.f;
  __syncwarp();
  const int Kb = pl.Kb[pa.i3];
  for (int u0 = 0; u0 < pa.c_in; u0 += 32) {
    const int u = u0 + lane;
    const bool active = u < pa.c_in;
    float G[RM][N3];
#pragma unroll
    for (int k = 0; k < RM; ++k)
#pragma unroll
      for (int i = 0; i < N3; ++i)
        G[k][i] = (active && k < pl.R) ? Gblk[size_t(rl * N3 + i) * Kb + pa.koff + k * pa.c_in + u] : 0.f;
    const float* xb = x + pa.in_off + size_t(active ? u : 0) * N1;
    for (int j = 0; j < nb; ++j) {
      const float* xp = xb + size_t(sS[j]) * pl.dim_in;
      float xv[N1];
#pragma unroll
      for (int i = 0; i < N1; ++i) xv[i] = active ? __ldg(xp + i) : 0.f;
      float T[N3];
      apply_M<L1, L2, L3>(sM + j * NMZ, xv, T);
      float red[N2 + RM];
      float dT[N3];
#pragma unroll
      for (int i = 0; i < N3; ++i) dT[i] = 0.f;
#pragma unroll
      for (int k = 0; k < RM; ++k) {
        const float bk = sB[j * RM + k];
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < N3; ++i) {
          dT[i] = fmaf(bk, G[k][i], dT[i]);
          s = fmaf(G[k][i], T[i], s);
        }
        red[N2 + k] = s;
      }
      cg_contract_13<L1, L2, L3>(xv, dT, red);
      warp_sum_all<N2 + RM>(red);
      if (lane == 0) {
#pragma unroll
        for (int i = 0; i < N2 + RM; ++i) sAcc[j * (N2 + RM) + i] += red[i];
      }
    }
  }
  __syncwarp();
}

template <int RM>
__device__ __forceinline__ void radj_dispatch(const DevPlan& pl, const DevPath& pa, int rl, int eb, int nb,
                                              const int* col, const float* vec, const float* x,
                                              const float* Gblk, float* sm) {
  switch (triple_id(pa.l1, pa.l2, pa.l3)) {
#define TPC_CASE(a, b, c)                                                \
  case triple_id(a, b, c):                                               \
    radj_path<a, b, c, RM>(pl, pa, rl, eb, nb, col, vec, x, Gblk, sm);   \
    break;
    TPC_FOR_EACH_TRIPLE(TPC_CASE)
#undef TPC_CASE
    default: break;
  }
}

// d_vec = grad_v [ sum_m dY[m] Y_m(v) + sum_k db[k] b_k(v) ]   (dual numbers)
template <int RM>
__device__ __forceinline__ void edge_vec_grad(const DevPlan& pl, const float* v, const float* dY,
                                              const float* db, float* out) {
  using D3 = Dual<float, 3>;
  D3 vx(v[0]), vy(v[1]), vz(v[2]);
  vx.d[0] = 1.f;
  vy.d[1] = 1.f;
  vz.d[2] = 1.f;
  D3 nx, ny, nz, r;
  unit(vx, vy, vz, nx, ny, nz, r);
  D3 Y[16];
  switch (pl.lsh) {
    case 0: sh_all<0>(nx, ny, nz, Y); break;
    case 1: sh_all<1>(nx, ny, nz, Y); break;
    case 2: sh_all<2>(nx, ny, nz, Y); break;
    default: sh_all<3>(nx, ny, nz, Y); break;
  }
  D3 b[RM];
  radial_basis<RM>(pl, r, b);
  float g0 = 0.f, g1 = 0.f, g2 = 0.f;
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    if (m >= pl.n_sh) break;
    g0 = fmaf(dY[m], Y[m].d[0], g0);
    g1 = fmaf(dY[m], Y[m].d[1], g1);
    g2 = fmaf(dY[m], Y[m].d[2], g2);
  }
#pragma unroll
  for (int k = 0; k < RM; ++k) {
    if (k >= pl.R) break;
    g0 = fmaf(db[k], b[k].d[0], g0);
    g1 = fmaf(db[k], b[k].d[1], g1);
    g2 = fmaf(db[k], b[k].d[2], g2);
  }
  out[0] = g0;
  out[1] = g1;
  out[2] = g2;
}

// grid: receivers in chunk; block: 32 * min(P, 16) (paths beyond 16 looped)
template <int RM>
__global__ void __launch_bounds__(512) k_radj_stream(const __grid_constant__ DevPlan pl, int r0, int nc,
                                                      const int* __restrict__ rowptr,
                                                      const int* __restrict__ col,
                                                      const float* __restrict__ vec,
                                                      const float* __restrict__ x,
                                                      const float* __restrict__ G, float* __restrict__ dvec,
                                                      float* __restrict__ dYout, float* __restrict__ dbout) {
  extern __shared__ float smem[];
  const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int rl = blockIdx.x;
  const int r = r0 + rl;
  const int e0 = rowptr[r], e1 = rowptr[r + 1];
  for (int eb = e0; eb < e1; eb += kEdgeBatch) {
    const int nb = min(kEdgeBatch, e1 - eb);
    for (int p = warp; p < pl.P; p += nwarps) {
      const DevPath& pa = pl.path[p];
      const float* Gblk = G + size_t(nc) * pl.a_pref[pa.i3];
      radj_dispatch<RM>(pl, pa, rl, eb, nb, col, vec, x, Gblk, smem + pa.sm_off);
    }
    __syncthreads();
    if (warp == 0 && lane_id() < nb) {
      const int j = lane_id();
      const int e = eb + j;
      float dY[16], db[RM];
#pragma unroll
      for (int m = 0; m < 16; ++m) dY[m] = 0.f;
#pragma unroll
      for (int k = 0; k < RM; ++k) db[k] = 0.f;
      for (int p = 0; p < pl.P; ++p) {
        const DevPath& pa = pl.path[p];
        const int N2 = 2 * pa.l2 + 1;
        const float* acc = smem + pa.sm_off + kEdgeBatch * (pa.nmz + RM + 1) + j * (N2 + RM);
        const int o = pa.l2 * pa.l2;
#pragma unroll
        for (int m = 0; m < 16; ++m)
          if (m >= o && m < o + N2) dY[m] += acc[m - o];
#pragma unroll
        for (int k = 0; k < RM; ++k) db[k] += acc[N2 + k];
      }
      float v[3] = {vec[3 * e], vec[3 * e + 1], vec[3 * e + 2]};
      if (dvec) {
        float o[3];
        edge_vec_grad<RM>(pl, v, dY, db, o);
        dvec[3 * e] = o[0];
        dvec[3 * e + 1] = o[1];
        dvec[3 * e + 2] = o[2];
      }
      if (dYout) {
#pragma unroll
        for (int m = 0; m < 16; ++m)
          if (m < pl.n_sh) dYout[size_t(e) * pl.n_sh + m] = dY[m];
      }
      if (dbout) {
#pragma unroll
        for (int k = 0; k < RM; ++k)
          if (k < pl.R) dbout[size_t(e) * pl.R + k] = db[k];
      }
    }
    __syncthreads();
  }
}

}  // namespace tpc
