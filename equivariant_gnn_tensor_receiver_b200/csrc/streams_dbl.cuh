// Double-backward edge streams.
//
// With Phi(g, x, Y, b, Theta) = <g, out> (linear in every slot), cotangents
// (gg_x, gg_vec, gg_theta) on (dx, dvec, dtheta), Ydot = J_Y gg_vec and
// bdot = J_b gg_vec, the second-order scalar is
//     Psi = Phi(g, gg_x, Y, b, Th) + Phi(g, x, Y, b, gg_Th)
//         + Phi(g, x, Ydot, b, Th) + Phi(g, x, Y, bdot, Th),
// and the abstract of "Sobek" (arXiv 2607.18074) states the streaming
// reassociation extends to this order.  Reassociated the same way as the first
// order, its derivatives need three streams:
//   k_dbl_a_path  receiver-sorted:  A1 = sum_e b (x) (M gg_x + Mdot x) + bdot (x) M x,
//                                   A0 = sum_e b (x) M x;   d_g = A1 Th + A0 gg_Th
//   k_dbl_s_path  sender-sorted:    B1 = sum_e b (x) Mdot^T g + bdot (x) M^T g,
//                                   B0 = sum_e b (x) M^T g; d_x = B1 Th + B0 gg_Th,
//                                   d_Th = x^T B1 + gg_x^T B0
//   k_dbl_r_stream receiver-sorted with G = Th^T g and Gt = gg_Th^T g resident:
//                 dPsi/db_k = <G_k, M gg_x + Mdot x> + <Gt_k, M x>,   db0_k = <G_k, M x>
//                 dPsi/dY   = C(gg_x, sum_k b_k G_k) + C(x, sum_k b_k Gt_k + bdot_k G_k),
//                 dY0       = C(x, sum_k b_k G_k)
//                 d_vec = grad_v [dPsi/dY . Y + dPsi/db . b + dY0 . Ydot + db0 . bdot]
// where Mdot is the coupling matrix of Ydot.  Null cotangents contribute zero
// (flags has_x1 = gg_x given, has_v = gg_vec given, has_t = gg_theta given).
#pragma once

#include "streams.cuh"

namespace tpc {

// Y, Ydot (degree L2) and b, bdot of one edge; directional derivative along u.
template <int L2, int RM>
__device__ __forceinline__ void geom_dir(const DevPlan& pl, const float* v, const float* u, float* Y, float* Yd,
                                         float* b, float* bd) {
  using D1 = Dual<float, 1>;
  D1 vx(v[0]), vy(v[1]), vz(v[2]);
  vx.d[0] = u[0];
  vy.d[0] = u[1];
  vz.d[0] = u[2];
  D1 nx, ny, nz, r;
  unit(vx, vy, vz, nx, ny, nz, r);
  D1 Yv[2 * L2 + 1];
  sh_degree<L2>(nx, ny, nz, Yv);
#pragma unroll
  for (int i = 0; i < 2 * L2 + 1; ++i) {
    Y[i] = Yv[i].v;
    Yd[i] = Yv[i].d[0];
  }
  D1 bv[RM];
  radial_basis<RM>(pl, r, bv);
#pragma unroll
  for (int k = 0; k < RM; ++k) {
    b[k] = bv[k].v;
    bd[k] = bv[k].d[0];
  }
}

// per-batch preparation (lane = edge): M, Mdot, b, bdot into warp scratch
template <int L1, int L2, int L3, int RM>
__device__ __forceinline__ void prep_edge_dir(const DevPlan& pl, const float* v, const float* u, float* sM,
                                              float* sMd, float* sB, float* sBd) {
  using TR = Tri<L1, L2, L3>;
  float Y[TR::N2], Yd[TR::N2], b[RM], bd[RM];
  geom_dir<L2, RM>(pl, v, u, Y, Yd, b, bd);
  const int lane = lane_id();
  coupling_row<L1, L2, L3>(Y, sM + lane * TR::NMZ);
  coupling_row<L1, L2, L3>(Yd, sMd + lane * TR::NMZ);
#pragma unroll
  for (int k = 0; k < RM; ++k) {
    sB[lane * RM + k] = b[k];
    sBd[lane * RM + k] = bd[k];
  }
}

__device__ __forceinline__ void load3(const float* p, int e, float* v) {
  v[0] = p[3 * e];
  v[1] = p[3 * e + 1];
  v[2] = p[3 * e + 2];
}

// ===========================================================================
// receiver stream -> [A1 | A0]
// ===========================================================================
template <int L1, int L2, int L3, int RM>
__global__ void __launch_bounds__(32 * kWarpsPerBlock)
    k_dbl_a_path(const __grid_constant__ DevPlan pl, int p, int r0, int nc, const int* __restrict__ rowptr,
                 const int* __restrict__ col, const float* __restrict__ vec, const float* __restrict__ ggv,
                 const float* __restrict__ x, const float* __restrict__ ggx, float* __restrict__ A1,
                 float* __restrict__ A0) {
  using TR = Tri<L1, L2, L3>;
  constexpr int N1 = TR::N1, N3 = TR::N3, NMZ = TR::NMZ, EB = kEdgeBatch;
  constexpr int WS = EB * (2 * NMZ + 2 * RM + 1);
  __shared__ float smem[kWarpsPerBlock * WS];
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const int rl = blockIdx.x * kWarpsPerBlock + warp;
  if (rl >= nc) return;
  const DevPath& pa = pl.path[p];
  float* sM = smem + warp * WS;
  float* sMd = sM + EB * NMZ;
  float* sB = sMd + EB * NMZ;
  float* sBd = sB + EB * RM;
  int* sS = reinterpret_cast<int*>(sBd + EB * RM);
  const int u = blockIdx.y * 32 + lane;
  const bool active = u < pa.c_in;
  float a1[RM][N3], a0[RM][N3];
#pragma unroll
  for (int k = 0; k < RM; ++k)
#pragma unroll
    for (int i = 0; i < N3; ++i) a1[k][i] = a0[k][i] = 0.f;
  const int r = r0 + rl;
  const int e0 = rowptr[r], e1 = rowptr[r + 1];
  const size_t cofs = pa.in_off + size_t(active ? u : 0) * N1;
  for (int eb = e0; eb < e1; eb += EB) {
    const int nb = min(EB, e1 - eb);
    __syncwarp();
    if (lane < nb) {
      const int e = eb + lane;
      float v[3], gv[3] = {0.f, 0.f, 0.f};
      load3(vec, e, v);
      if (ggv) load3(ggv, e, gv);
      prep_edge_dir<L1, L2, L3, RM>(pl, v, gv, sM, sMd, sB, sBd);
      sS[lane] = col[e];
    }
    __syncwarp();
    for (int j = 0; j < nb; ++j) {
      const size_t ro = size_t(sS[j]) * pl.dim_in + cofs;
      float xv[N1], gx[N1];
#pragma unroll
      for (int i = 0; i < N1; ++i) {
        xv[i] = active ? __ldg(x + ro + i) : 0.f;
        gx[i] = (active && ggx) ? __ldg(ggx + ro + i) : 0.f;
      }
      float T0[N3], T1[N3], T2[N3];
      apply_M<L1, L2, L3>(sM + j * NMZ, xv, T0);
      apply_M<L1, L2, L3>(sM + j * NMZ, gx, T1);
      apply_M<L1, L2, L3>(sMd + j * NMZ, xv, T2);
#pragma unroll
      for (int k = 0; k < RM; ++k) {
        const float bk = sB[j * RM + k], bdk = sBd[j * RM + k];
#pragma unroll
        for (int i = 0; i < N3; ++i) {
          a0[k][i] = fmaf(bk, T0[i], a0[k][i]);
          a1[k][i] = fmaf(bk, T1[i] + T2[i], fmaf(bdk, T0[i], a1[k][i]));
        }
      }
    }
  }
  if (!active) return;
  const int Kb = pl.Kb[pa.i3];
  const size_t base = size_t(nc) * pl.a_pref[pa.i3];
#pragma unroll
  for (int k = 0; k < RM; ++k) {
    if (k >= pl.R) break;
#pragma unroll
    for (int i = 0; i < N3; ++i) {
      const size_t o = base + size_t(rl * N3 + i) * Kb + pa.koff + k * pa.c_in + u;
      A1[o] = a1[k][i];
      A0[o] = a0[k][i];
    }
  }
}

// ===========================================================================
// sender stream -> [B1 | B0]
// ===========================================================================
template <int L1, int L2, int L3, int RM>
__global__ void __launch_bounds__(32 * kWarpsPerBlock)
    k_dbl_s_path(const __grid_constant__ DevPlan pl, int p, int s0, int nc, const int* __restrict__ s_rowptr,
                 const int* __restrict__ perm, const int* __restrict__ s_recv, const float* __restrict__ vec,
                 const float* __restrict__ ggv, const float* __restrict__ g, float* __restrict__ B1,
                 float* __restrict__ B0) {
  using TR = Tri<L1, L2, L3>;
  constexpr int N1 = TR::N1, N3 = TR::N3, NMZ = TR::NMZ, EB = kEdgeBatch;
  constexpr int WS = EB * (2 * NMZ + 2 * RM + 1);
  __shared__ float smem[kWarpsPerBlock * WS];
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const int sl = blockIdx.x * kWarpsPerBlock + warp;
  if (sl >= nc) return;
  const DevPath& pa = pl.path[p];
  float* sM = smem + warp * WS;
  float* sMd = sM + EB * NMZ;
  float* sB = sMd + EB * NMZ;
  float* sBd = sB + EB * RM;
  int* sR = reinterpret_cast<int*>(sBd + EB * RM);
  const int w = blockIdx.y * 32 + lane;
  const bool active = w < pa.c_out;
  float b1[RM][N1], b0[RM][N1];
#pragma unroll
  for (int k = 0; k < RM; ++k)
#pragma unroll
    for (int i = 0; i < N1; ++i) b1[k][i] = b0[k][i] = 0.f;
  const int s = s0 + sl;
  const int j0 = s_rowptr[s], j1 = s_rowptr[s + 1];
  const float* gb = g + pa.out_off + size_t(active ? w : 0) * N3;
  for (int jb = j0; jb < j1; jb += EB) {
    const int nb = min(EB, j1 - jb);
    __syncwarp();
    if (lane < nb) {
      const int e = perm[jb + lane];
      float v[3], gv[3] = {0.f, 0.f, 0.f};
      load3(vec, e, v);
      if (ggv) load3(ggv, e, gv);
      prep_edge_dir<L1, L2, L3, RM>(pl, v, gv, sM, sMd, sB, sBd);
      sR[lane] = s_recv[jb + lane];
    }
    __syncwarp();
    for (int j = 0; j < nb; ++j) {
      const float* gp = gb + size_t(sR[j]) * pl.dim_out;
      float gv[N3];
#pragma unroll
      for (int i = 0; i < N3; ++i) gv[i] = active ? __ldg(gp + i) : 0.f;
      float U0[N1], U1[N1];
      apply_Mt<L1, L2, L3>(sM + j * NMZ, gv, U0);
      apply_Mt<L1, L2, L3>(sMd + j * NMZ, gv, U1);
#pragma unroll
      for (int k = 0; k < RM; ++k) {
        const float bk = sB[j * RM + k], bdk = sBd[j * RM + k];
#pragma unroll
        for (int i = 0; i < N1; ++i) {
          b0[k][i] = fmaf(bk, U0[i], b0[k][i]);
          b1[k][i] = fmaf(bk, U1[i], fmaf(bdk, U0[i], b1[k][i]));
        }
      }
    }
  }
  if (!active) return;
  const int Kx = pl.Kx[pa.i1];
  const size_t base = size_t(nc) * pl.b_pref[pa.i1];
#pragma unroll
  for (int k = 0; k < RM; ++k) {
    if (k >= pl.R) break;
#pragma unroll
    for (int i = 0; i < N1; ++i) {
      const size_t o = base + size_t(sl * N1 + i) * Kx + pa.kxoff + k * pa.c_out + w;
      B1[o] = b1[k][i];
      B0[o] = b0[k][i];
    }
  }
}

// ===========================================================================
// receiver adjoint stream -> d_vec
// ===========================================================================
// Per-edge accumulator layout of one path: [dPsi/dY (N2) | dY0 (N2) | dPsi/db (RM) | db0 (RM)]
template <int L1, int L2, int L3, int RM>
__device__ __forceinline__ void dbl_r_path(const DevPlan& pl, const DevPath& pa, int rl, int eb, int nb,
                                           const int* __restrict__ col, const float* __restrict__ vec,
                                           const float* __restrict__ ggv, const float* __restrict__ x,
                                           const float* __restrict__ ggx, const float* __restrict__ Gblk,
                                           const float* __restrict__ Gtblk, float* sm) {
  using TR = Tri<L1, L2, L3>;
  constexpr int N1 = TR::N1, N2 = TR::N2, N3 = TR::N3, NMZ = TR::NMZ, EB = kEdgeBatch;
  constexpr int NA = 2 * N2 + 2 * RM;
  float* sM = sm;
  float* sMd = sM + EB * NMZ;
  float* sB = sMd + EB * NMZ;
  float* sBd = sB + EB * RM;
  int* sS = reinterpret_cast<int*>(sBd + EB * RM);
  float* sAcc = reinterpret_cast<float*>(sS + EB);  // [EB][NA]
  const int lane = lane_id();
  __syncwarp();
  if (lane < nb) {
    const int e = eb + lane;
    float v[3], gv[3] = {0.f, 0.f, 0.f};
    load3(vec, e, v);
    if (ggv) load3(ggv, e, gv);
    prep_edge_dir<L1, L2, L3, RM>(pl, v, gv, sM, sMd, sB, sBd);
    sS[lane] = col[e];
  }
  for (int i = lane; i < EB * NA; i += 32) sAcc[i] = 0.f;
  __syncwarp();
  const int Kb = pl.Kb[pa.i3];
  for (int u0 = 0; u0 < pa.c_in; u0 += 32) {
    const int u = u0 + lane;
    const bool active = u < pa.c_in;
    float G[RM][N3], Gt[RM][N3];
#pragma unroll
    for (int k = 0; k < RM; ++k)
#pragma unroll
      for (int i = 0; i < N3; ++i) {
        const size_t o = size_t(rl * N3 + i) * Kb + pa.koff + k * pa.c_in + u;
        const bool ok = active && k < pl.R;
        G[k][i] = ok ? Gblk[o] : 0.f;
        Gt[k][i] = (ok && Gtblk) ? Gtblk[o] : 0.f;
      }
    const size_t cofs = pa.in_off + size_t(active ? u : 0) * N1;
    for (int j = 0; j < nb; ++j) {
      const size_t ro = size_t(sS[j]) * pl.dim_in + cofs;
      float xv[N1], gx[N1];
#pragma unroll
      for (int i = 0; i < N1; ++i) {
        xv[i] = active ? __ldg(x + ro + i) : 0.f;
        gx[i] = (active && ggx) ? __ldg(ggx + ro + i) : 0.f;
      }
      float T0[N3], T12[N3];
      apply_M<L1, L2, L3>(sM + j * NMZ, xv, T0);
      {
        float T1[N3], T2[N3];
        apply_M<L1, L2, L3>(sM + j * NMZ, gx, T1);
        apply_M<L1, L2, L3>(sMd + j * NMZ, xv, T2);
#pragma unroll
        for (int i = 0; i < N3; ++i) T12[i] = T1[i] + T2[i];
      }
      float red[NA];
      float dG[N3], dX[N3];  // dG = sum b G ; dX = sum b Gt + bdot G
#pragma unroll
      for (int i = 0; i < N3; ++i) dG[i] = dX[i] = 0.f;
#pragma unroll
      for (int k = 0; k < RM; ++k) {
        const float bk = sB[j * RM + k], bdk = sBd[j * RM + k];
        float s1 = 0.f, s0 = 0.f;
#pragma unroll
        for (int i = 0; i < N3; ++i) {
          dG[i] = fmaf(bk, G[k][i], dG[i]);
          dX[i] = fmaf(bk, Gt[k][i], fmaf(bdk, G[k][i], dX[i]));
          s1 = fmaf(G[k][i], T12[i], fmaf(Gt[k][i], T0[i], s1));
          s0 = fmaf(G[k][i], T0[i], s0);
        }
        red[2 * N2 + k] = s1;
        red[2 * N2 + RM + k] = s0;
      }
      float t1[N2], t2[N2];
      cg_contract_13<L1, L2, L3>(gx, dG, t1);
      cg_contract_13<L1, L2, L3>(xv, dX, t2);
      cg_contract_13<L1, L2, L3>(xv, dG, red + N2);
#pragma unroll
      for (int i = 0; i < N2; ++i) red[i] = t1[i] + t2[i];
      warp_sum_all<NA>(red);
      if (lane == 0) {
#pragma unroll
        for (int i = 0; i < NA; ++i) sAcc[j * NA + i] += red[i];
      }
    }
  }
  __syncwarp();
}

template <int RM>
__device__ __forceinline__ void dbl_r_dispatch(const DevPlan& pl, const DevPath& pa, int rl, int eb, int nb,
                                               const int* col, const float* vec, const float* ggv, const float* x,
                                               const float* ggx, const float* Gblk, const float* Gtblk,
                                               float* sm) {
  switch (triple_id(pa.l1, pa.l2, pa.l3)) {
#define TPC_CASE(a, b, c)                                                                     \
  case triple_id(a, b, c):                                                                    \
    dbl_r_path<a, b, c, RM>(pl, pa, rl, eb, nb, col, vec, ggv, x, ggx, Gblk, Gtblk, sm);     \
    break;
    TPC_FOR_EACH_TRIPLE(TPC_CASE)
#undef TPC_CASE
    default: break;
  }
}

// d_vec = grad_v [ sum_m (wY[m] Y_m + hY[m] dY_m/du) + sum_k (wb[k] b_k + hb[k] db_k/du) ]
template <int RM>
__device__ __forceinline__ void edge_vec_grad2(const DevPlan& pl, const float* v, const float* u, const float* wY,
                                               const float* hY, const float* wb, const float* hb, float* out) {
  using D1 = Dual<float, 1>;
  using DD = Dual<D1, 3>;
  DD c[3];
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    c[i] = DD(0.f);
    c[i].v.v = v[i];
    c[i].v.d[0] = u[i];
    c[i].d[i].v = 1.f;
  }
  DD nx, ny, nz, r;
  unit(c[0], c[1], c[2], nx, ny, nz, r);
  float g[3] = {0.f, 0.f, 0.f};
  // one SH degree at a time keeps the nested duals of only 2l+1 harmonics live
  auto degree = [&](auto LC) {
    constexpr int L = decltype(LC)::value;
    if (L > pl.lsh) return;
    DD Y[2 * L + 1];
    sh_degree<L>(nx, ny, nz, Y);
#pragma unroll
    for (int i = 0; i < 2 * L + 1; ++i) {
      const int m = L * L + i;
#pragma unroll
      for (int a = 0; a < 3; ++a) g[a] = fmaf(wY[m], Y[i].d[a].v, fmaf(hY[m], Y[i].d[a].d[0], g[a]));
    }
  };
  degree(std::integral_constant<int, 0>{});
  degree(std::integral_constant<int, 1>{});
  degree(std::integral_constant<int, 2>{});
  degree(std::integral_constant<int, 3>{});
  DD b[RM];
  radial_basis<RM>(pl, r, b);
#pragma unroll
  for (int k = 0; k < RM; ++k) {
    if (k >= pl.R) break;
#pragma unroll
    for (int i = 0; i < 3; ++i) g[i] = fmaf(wb[k], b[k].d[i].v, fmaf(hb[k], b[k].d[i].d[0], g[i]));
  }
  out[0] = g[0];
  out[1] = g[1];
  out[2] = g[2];
}

template <int RM>
__global__ void __launch_bounds__(512) k_dbl_r_stream(const __grid_constant__ DevPlan pl, int r0, int nc,
                                                      const int* __restrict__ rowptr, const int* __restrict__ col,
                                                      const float* __restrict__ vec, const float* __restrict__ ggv,
                                                      const float* __restrict__ x, const float* __restrict__ ggx,
                                                      const float* __restrict__ G, const float* __restrict__ Gt,
                                                      float* __restrict__ dvec) {
  extern __shared__ float smem[];
  const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int rl = blockIdx.x;
  const int r = r0 + rl;
  const int e0 = rowptr[r], e1 = rowptr[r + 1];
  for (int eb = e0; eb < e1; eb += kEdgeBatch) {
    const int nb = min(kEdgeBatch, e1 - eb);
    for (int p = warp; p < pl.P; p += nwarps) {
      const DevPath& pa = pl.path[p];
      const size_t off = size_t(nc) * pl.a_pref[pa.i3];
      dbl_r_dispatch<RM>(pl, pa, rl, eb, nb, col, vec, ggv, x, ggx, G + off, Gt ? Gt + off : nullptr,
                         smem + pa.sm_off2);
    }
    __syncthreads();
    if (warp == 0 && lane_id() < nb) {
      const int j = lane_id();
      const int e = eb + j;
      float wY[16], hY[16], wb[RM], hb[RM];
#pragma unroll
      for (int m = 0; m < 16; ++m) wY[m] = hY[m] = 0.f;
#pragma unroll
      for (int k = 0; k < RM; ++k) wb[k] = hb[k] = 0.f;
      for (int p = 0; p < pl.P; ++p) {
        const DevPath& pa = pl.path[p];
        const int N2 = 2 * pa.l2 + 1, NA = 2 * N2 + 2 * RM;
        const float* acc = smem + pa.sm_off2 + kEdgeBatch * (2 * pa.nmz + 2 * RM + 1) + j * NA;
        const int o = pa.l2 * pa.l2;
#pragma unroll
        for (int m = 0; m < 16; ++m)
          if (m >= o && m < o + N2) {
            wY[m] += acc[m - o];
            hY[m] += acc[N2 + m - o];
          }
#pragma unroll
        for (int k = 0; k < RM; ++k) {
          wb[k] += acc[2 * N2 + k];
          hb[k] += acc[2 * N2 + RM + k];
        }
      }
      float v[3], u[3] = {0.f, 0.f, 0.f}, o3[3];
      load3(vec, e, v);
      if (ggv) load3(ggv, e, u);
      edge_vec_grad2<RM>(pl, v, u, wY, hY, wb, hb, o3);
      dvec[3 * e] = o3[0];
      dvec[3 * e + 1] = o3[1];
      dvec[3 * e + 2] = o3[2];
    }
    __syncthreads();
  }
}

}  // namespace tpc
