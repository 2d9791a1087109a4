// Path-major receiver adjoint streams (first and second order), lane = edge.
//
// All warps of a CTA work on the same path at the same time: the paths are
// iterated uniformly, each path's code is executed by every warp (one hot body
// in the instruction cache, no per-path load imbalance between warps), and the
// warps split the path's channels.  A lane owns one edge of the batch and keeps
// that edge's adjoint accumulators in registers across all paths; one
// cross-warp reduction per edge batch combines the channel slices.
//
// First order (per edge e = (s -> r), G = Theta^T g_r):
//     db_ek = sum_{p,u,m3} G[k,p,u,m3] (M_e x_s)[p,u,m3]
//     dY_e  = sum_p sum_u C_p(x_s[u], sum_k b_ek G[k,p,u])
//     dvec_e = J_Y^T dY_e + J_b^T db_e
// Second order (Gt = gg_Theta^T g_r, Mdot / bdot along gg_vec_e): see
// streams_dbl.cuh for the four accumulators (dPsi/dY, dY0, dPsi/db, db0) and
//     d_vec_e = grad_v [dPsi/dY . Y + dPsi/db . b + dY0 . Ydot + db0 . bdot].
//
// Backward of the streaming schedule ("Sobek", arXiv 2607.18074, abstract).
#pragma once

#include "pm_layout.h"
#include "streams_dbl.cuh"
#include "streams_v2.cuh"

namespace tpc {

// stage, for one path and channel tile [c0, c0+w): G (and Gt) as [k][m3][c] with
// row stride L.tile, and the batch's rows of input block i1 (x, and x1) as
// [edge][c * n1 + m1] with row stride xs.  All threads; ends with a barrier.
__device__ __forceinline__ void pm_stage(const DevPlan& pl, const DevPath& q, const PmLay& L, float* sm, int rl, int nb,
                                         int c0, int w, const float* __restrict__ G, const float* __restrict__ Gt,
                                         int nc, const float* __restrict__ x, const float* __restrict__ x1) {
  const int n3 = 2 * q.l3 + 1, n1 = 2 * q.l1 + 1, Kb = pl.Kb[q.i3];
  const int w4 = w >> 2;
  const size_t goff = size_t(nc) * pl.a_pref[q.i3] + size_t(rl) * n3 * Kb + q.koff + c0;
  const int tg = pl.R * n3 * w4;
  for (int idx = threadIdx.x; idx < tg; idx += blockDim.x) {
    const int row = idx / w4, c = idx - row * w4;  // row = k * n3 + m3
    const int k = row / n3, m3 = row - k * n3;
    const size_t src = goff + size_t(m3) * Kb + size_t(k) * q.c_in + 4 * c;
    cp_async16(sm + L.G + row * L.tile + 4 * c, G + src);
    if (Gt) cp_async16(sm + L.Gt + row * L.tile + 4 * c, Gt + src);
  }
  const int* scol = reinterpret_cast<const int*>(sm + L.S);
  const int len = w * n1;
  const int so = q.in_off + c0 * n1;
  for (int j = 0; j < nb; ++j) {
    const size_t rb = size_t(scol[j]) * pl.dim_in + so;
    for (int o = threadIdx.x; o < len; o += blockDim.x) {
      cp_async4(sm + L.X + j * L.xs + o, x + rb + o);
      if (x1) cp_async4(sm + L.X1 + j * L.xs + o, x1 + rb + o);
    }
  }
  cp_async_commit();
  cp_async_wait_all();
  __syncthreads();
}

// ---- first order: one path, this warp's channels of the staged tile --------
template <int L1, int L2, int L3, int RM>
__device__ __forceinline__ void pm_adj_body(const PmLay& L, const float* sm, int lane, int u0, int u1,
                                            float* dY, float* db) {
  using TR = Tri<L1, L2, L3>;
  constexpr int N1 = TR::N1, N2 = TR::N2, N3 = TR::N3, NMZ = TR::NMZ;
  float Mv[NMZ > 0 ? NMZ : 1], bv[RM];
  coupling_row<L1, L2, L3>(sm + L.Y + lane * 16 + L2 * L2, Mv);
#pragma unroll
  for (int k = 0; k < RM; ++k) bv[k] = sm[L.B + lane * RM + k];
  const float* xr = sm + L.X + lane * L.xs;
  float dYl[N2];
#pragma unroll
  for (int i = 0; i < N2; ++i) dYl[i] = 0.f;
  for (int u = u0; u < u1; ++u) {
    float xv[N1], T[N3], dT[N3];
#pragma unroll
    for (int i = 0; i < N1; ++i) xv[i] = xr[u * N1 + i];
    apply_M<L1, L2, L3>(Mv, xv, T);
#pragma unroll
    for (int i = 0; i < N3; ++i) dT[i] = 0.f;
#pragma unroll
    for (int k = 0; k < RM; ++k) {
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < N3; ++i) {
        const float g = sm[L.G + (k * N3 + i) * L.tile + u];
        dT[i] = fmaf(bv[k], g, dT[i]);
        s = fmaf(g, T[i], s);
      }
      db[k] += s;
    }
    float t[N2];
    cg_contract_13<L1, L2, L3>(xv, dT, t);
#pragma unroll
    for (int i = 0; i < N2; ++i) dYl[i] += t[i];
  }
#pragma unroll
  for (int i = 0; i < N2; ++i) dY[L2 * L2 + i] += dYl[i];
}

// ---- second order: one path, this warp's channels of the staged tile -------
template <int L1, int L2, int L3, int RM>
__device__ __forceinline__ void pm_dadj_body(const PmLay& L, const float* sm, int lane, int u0, int u1, bool has_x1,
                                             bool has_t, float* wY, float* hY, float* wb, float* hb) {
  using TR = Tri<L1, L2, L3>;
  constexpr int N1 = TR::N1, N2 = TR::N2, N3 = TR::N3, NMZ = TR::NMZ;
  float Mv[NMZ > 0 ? NMZ : 1], Mdv[NMZ > 0 ? NMZ : 1], bv[RM], bdv[RM];
  coupling_row<L1, L2, L3>(sm + L.Y + lane * 16 + L2 * L2, Mv);
  coupling_row<L1, L2, L3>(sm + L.Yd + lane * 16 + L2 * L2, Mdv);
#pragma unroll
  for (int k = 0; k < RM; ++k) {
    bv[k] = sm[L.B + lane * RM + k];
    bdv[k] = sm[L.Bd + lane * RM + k];
  }
  const float* xr = sm + L.X + lane * L.xs;
  const float* x1r = sm + L.X1 + lane * L.xs;
  float wYl[N2], hYl[N2];
#pragma unroll
  for (int i = 0; i < N2; ++i) wYl[i] = hYl[i] = 0.f;
  for (int u = u0; u < u1; ++u) {
    float xv[N1], x1[N1], T0[N3], T12[N3], dG[N3], dX[N3];
#pragma unroll
    for (int i = 0; i < N1; ++i) {
      xv[i] = xr[u * N1 + i];
      x1[i] = has_x1 ? x1r[u * N1 + i] : 0.f;
    }
    apply_M<L1, L2, L3>(Mv, xv, T0);
    {
      float ta[N3], tb[N3];
      apply_M<L1, L2, L3>(Mv, x1, ta);
      apply_M<L1, L2, L3>(Mdv, xv, tb);
#pragma unroll
      for (int i = 0; i < N3; ++i) T12[i] = ta[i] + tb[i];
    }
#pragma unroll
    for (int i = 0; i < N3; ++i) dG[i] = dX[i] = 0.f;
#pragma unroll
    for (int k = 0; k < RM; ++k) {
      float s1 = 0.f, s0 = 0.f;
#pragma unroll
      for (int i = 0; i < N3; ++i) {
        const float g = sm[L.G + (k * N3 + i) * L.tile + u];
        const float gt = has_t ? sm[L.Gt + (k * N3 + i) * L.tile + u] : 0.f;
        dG[i] = fmaf(bv[k], g, dG[i]);
        dX[i] = fmaf(bv[k], gt, fmaf(bdv[k], g, dX[i]));
        s1 = fmaf(g, T12[i], fmaf(gt, T0[i], s1));
        s0 = fmaf(g, T0[i], s0);
      }
      wb[k] += s1;
      hb[k] += s0;
    }
    float t1[N2], t2[N2], t3[N2];
    cg_contract_13<L1, L2, L3>(x1, dG, t1);
    cg_contract_13<L1, L2, L3>(xv, dX, t2);
    cg_contract_13<L1, L2, L3>(xv, dG, t3);
#pragma unroll
    for (int i = 0; i < N2; ++i) {
      wYl[i] += t1[i] + t2[i];
      hYl[i] += t3[i];
    }
  }
#pragma unroll
  for (int i = 0; i < N2; ++i) {
    wY[L2 * L2 + i] += wYl[i];
    hY[L2 * L2 + i] += hYl[i];
  }
}

// geometry of one batch (warp 0, lane = edge): Y, b (and Ydot, bdot along gg_vec)
template <int RM>
__device__ __forceinline__ void pm_geometry(const DevPlan& pl, const PmLay& L, float* sm, int eb, int nb,
                                            const int* __restrict__ col, const float* __restrict__ vec,
                                            const float* __restrict__ ggv, bool dir) {
  const int lane = lane_id();
  if ((threadIdx.x >> 5) != 0 || lane >= nb) return;
  const int e = eb + lane;
  using D1 = Dual<float, 1>;
  D1 vx(vec[3 * e]), vy(vec[3 * e + 1]), vz(vec[3 * e + 2]);
  if (dir && ggv) {
    vx.d[0] = ggv[3 * e];
    vy.d[0] = ggv[3 * e + 1];
    vz.d[0] = ggv[3 * e + 2];
  }
  D1 nx, ny, nz, rr;
  unit(vx, vy, vz, nx, ny, nz, rr);
  D1 Y[16], b[RM];
  switch (pl.lsh) {
    case 0: sh_all<0>(nx, ny, nz, Y); break;
    case 1: sh_all<1>(nx, ny, nz, Y); break;
    case 2: sh_all<2>(nx, ny, nz, Y); break;
    default: sh_all<3>(nx, ny, nz, Y); break;
  }
  radial_basis<RM>(pl, rr, b);
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    if (m >= pl.n_sh) break;
    sm[L.Y + lane * 16 + m] = Y[m].v;
    sm[L.Yd + lane * 16 + m] = Y[m].d[0];
  }
#pragma unroll
  for (int k = 0; k < RM; ++k) {
    sm[L.B + lane * RM + k] = b[k].v;
    sm[L.Bd + lane * RM + k] = b[k].d[0];
  }
  reinterpret_cast<int*>(sm + L.S)[lane] = col[e];
}

// channels of the tile [c0, c0+w) handled by warp `warp`
__device__ __forceinline__ void pm_slice(int w, int warp, int& u0, int& u1) {
  const int per = (w + kPmWarps - 1) / kPmWarps;
  u0 = min(w, warp * per);
  u1 = min(w, u0 + per);
}

// ---------------------------------------------------------------------------
// first order: grid = receivers in chunk, block = 32 * kPmWarps
// ---------------------------------------------------------------------------
template <int RM>
__global__ void __launch_bounds__(32 * kPmWarps, 2)
    k_pm_adj(const __grid_constant__ DevPlan pl, int r0, int nc, const int* __restrict__ rowptr,
             const int* __restrict__ col, const float* __restrict__ vec, const float* __restrict__ x,
             const float* __restrict__ G, float* __restrict__ dvec, float* __restrict__ dYout,
             float* __restrict__ dbout) {
  extern __shared__ __align__(16) float sm[];
  const PmLay L = pm_layout_of(RM, pl.pm_tile_a, pl.pm_n3max, pl.pm_n1max, pl.R, false);
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const int rl = blockIdx.x, r = r0 + rl;
  const int e0 = rowptr[r], e1 = rowptr[r + 1];
  for (int eb = e0; eb < e1; eb += kPmBatch) {
    const int nb = min(kPmBatch, e1 - eb);
    pm_geometry<RM>(pl, L, sm, eb, nb, col, vec, nullptr, false);
    __syncthreads();
    float dY[16], db[RM];
#pragma unroll
    for (int m = 0; m < 16; ++m) dY[m] = 0.f;
#pragma unroll
    for (int k = 0; k < RM; ++k) db[k] = 0.f;
    for (int p = 0; p < pl.P; ++p) {
      const DevPath& q = pl.path[p];
      for (int c0 = 0; c0 < q.c_in; c0 += L.tile) {
        const int w = min(L.tile, q.c_in - c0);
        pm_stage(pl, q, L, sm, rl, nb, c0, w, G, nullptr, nc, x, nullptr);
        int u0, u1;
        pm_slice(w, warp, u0, u1);
        if (lane < nb && u0 < u1) {
          switch (triple_id(q.l1, q.l2, q.l3)) {
#define TPC_CASE(a, b, c)                                                \
  case triple_id(a, b, c):                                               \
    pm_adj_body<a, b, c, RM>(L, sm, lane, u0, u1, dY, db);               \
    break;
            TPC_FOR_EACH_TRIPLE(TPC_CASE)
#undef TPC_CASE
            default: break;
          }
        }
        __syncthreads();
      }
    }
    // combine the warps' channel slices per edge
    float* red = sm + L.Red + (warp * kPmBatch + lane) * (16 + RM);
#pragma unroll
    for (int m = 0; m < 16; ++m) red[m] = dY[m];
#pragma unroll
    for (int k = 0; k < RM; ++k) red[16 + k] = db[k];
    __syncthreads();
    if (warp == 0 && lane < nb) {
      const int e = eb + lane;
      float sY[16], sb[RM];
#pragma unroll
      for (int m = 0; m < 16; ++m) sY[m] = 0.f;
#pragma unroll
      for (int k = 0; k < RM; ++k) sb[k] = 0.f;
      for (int w = 0; w < kPmWarps; ++w) {
        const float* rr = sm + L.Red + (w * kPmBatch + lane) * (16 + RM);
#pragma unroll
        for (int m = 0; m < 16; ++m) sY[m] += rr[m];
#pragma unroll
        for (int k = 0; k < RM; ++k) sb[k] += rr[16 + k];
      }
      if (dvec) {
        const float v[3] = {vec[3 * e], vec[3 * e + 1], vec[3 * e + 2]};
        float o3[3];
        edge_vec_grad<RM>(pl, v, sY, sb, o3);
        dvec[3 * e] = o3[0];
        dvec[3 * e + 1] = o3[1];
        dvec[3 * e + 2] = o3[2];
      }
      if (dYout) {
#pragma unroll
        for (int m = 0; m < 16; ++m)
          if (m < pl.n_sh) dYout[size_t(e) * pl.n_sh + m] = sY[m];
      }
      if (dbout) {
#pragma unroll
        for (int k = 0; k < RM; ++k)
          if (k < pl.R) dbout[size_t(e) * pl.R + k] = sb[k];
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// second order: grid = receivers in chunk, block = 32 * kPmWarps
// ---------------------------------------------------------------------------
template <int RM>
__global__ void __launch_bounds__(32 * kPmWarps, 2)
    k_pm_dadj(const __grid_constant__ DevPlan pl, int r0, int nc, const int* __restrict__ rowptr,
              const int* __restrict__ col, const float* __restrict__ vec, const float* __restrict__ ggv,
              const float* __restrict__ x, const float* __restrict__ ggx, const float* __restrict__ G,
              const float* __restrict__ Gt, float* __restrict__ dvec) {
  extern __shared__ __align__(16) float sm[];
  const PmLay L = pm_layout_of(RM, pl.pm_tile_d, pl.pm_n3max, pl.pm_n1max, pl.R, true);
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const int rl = blockIdx.x, r = r0 + rl;
  const int e0 = rowptr[r], e1 = rowptr[r + 1];
  const bool has_x1 = ggx != nullptr, has_t = Gt != nullptr;
  for (int eb = e0; eb < e1; eb += kPmBatch) {
    const int nb = min(kPmBatch, e1 - eb);
    pm_geometry<RM>(pl, L, sm, eb, nb, col, vec, ggv, true);
    __syncthreads();
    float wY[16], hY[16], wb[RM], hb[RM];
#pragma unroll
    for (int m = 0; m < 16; ++m) wY[m] = hY[m] = 0.f;
#pragma unroll
    for (int k = 0; k < RM; ++k) wb[k] = hb[k] = 0.f;
    for (int p = 0; p < pl.P; ++p) {
      const DevPath& q = pl.path[p];
      for (int c0 = 0; c0 < q.c_in; c0 += L.tile) {
        const int w = min(L.tile, q.c_in - c0);
        pm_stage(pl, q, L, sm, rl, nb, c0, w, G, Gt, nc, x, ggx);
        int u0, u1;
        pm_slice(w, warp, u0, u1);
        if (lane < nb && u0 < u1) {
          switch (triple_id(q.l1, q.l2, q.l3)) {
#define TPC_CASE(a, b, c)                                                                   \
  case triple_id(a, b, c):                                                                  \
    pm_dadj_body<a, b, c, RM>(L, sm, lane, u0, u1, has_x1, has_t, wY, hY, wb, hb);          \
    break;
            TPC_FOR_EACH_TRIPLE(TPC_CASE)
#undef TPC_CASE
            default: break;
          }
        }
        __syncthreads();
      }
    }
    float* red = sm + L.Red + (warp * kPmBatch + lane) * (32 + 2 * RM);
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      red[m] = wY[m];
      red[16 + m] = hY[m];
    }
#pragma unroll
    for (int k = 0; k < RM; ++k) {
      red[32 + k] = wb[k];
      red[32 + RM + k] = hb[k];
    }
    __syncthreads();
    if (warp == 0 && lane < nb) {
      const int e = eb + lane;
      float sY[16], sH[16], sb[RM], sh[RM];
#pragma unroll
      for (int m = 0; m < 16; ++m) sY[m] = sH[m] = 0.f;
#pragma unroll
      for (int k = 0; k < RM; ++k) sb[k] = sh[k] = 0.f;
      for (int w = 0; w < kPmWarps; ++w) {
        const float* rr = sm + L.Red + (w * kPmBatch + lane) * (32 + 2 * RM);
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          sY[m] += rr[m];
          sH[m] += rr[16 + m];
        }
#pragma unroll
        for (int k = 0; k < RM; ++k) {
          sb[k] += rr[32 + k];
          sh[k] += rr[32 + RM + k];
        }
      }
      float v[3], u[3] = {0.f, 0.f, 0.f}, o3[3];
      load3(vec, e, v);
      if (ggv) load3(ggv, e, u);
      edge_vec_grad2<RM>(pl, v, u, sY, sH, sb, sh, o3);
      dvec[3 * e] = o3[0];
      dvec[3 * e + 1] = o3[1];
      dvec[3 * e + 2] = o3[2];
    }
    __syncthreads();
  }
}

}  // namespace tpc
