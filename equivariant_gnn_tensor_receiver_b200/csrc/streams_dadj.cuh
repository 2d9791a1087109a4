// Double-backward receiver adjoint stream with lane = edge.
//
// Per edge e = (s -> r), with T0 = M x_s, T12 = M gg_x_s + Mdot x_s (Mdot: the
// coupling matrix of Ydot = J_Y gg_vec_e), G = Theta^T g_r, Gt = gg_Theta^T g_r:
//     dPsi/db_k = <G_k, T12> + <Gt_k, T0>        db0_k = <G_k, T0>
//     dPsi/dY   = C(gg_x_s, sum_k b_k G_k) + C(x_s, sum_k (b_k Gt_k + bdot_k G_k))
//     dY0       = C(x_s, sum_k b_k G_k)
//     d_vec     = grad_v [dPsi/dY . Y + dPsi/db . b + dY0 . Ydot + db0 . bdot]
// (derivation in streams_dbl.cuh).  As in the first-order adjoint stream each
// lane owns one edge and keeps its four accumulators in registers; the channel
// tile of G (and Gt when gg_Theta is given) is staged in shared memory and read
// as warp-wide broadcasts, and x_s, gg_x_s rows are staged per batch of 32 edges
// with an odd row stride.
#pragma once

#include "streams_adj.cuh"
#include "streams_dbl.cuh"

namespace tpc {

struct DadjLay {
  int G, Gt, X, X1, Y, Yd, B, Bd, S, Acc;
  int xs;
};

__device__ __forceinline__ DadjLay dadj_layout(const DevPlan& pl, int RM) {
  DadjLay L;
  L.G = 0;
  L.Gt = L.G + pl.dadj_g;
  L.X = L.Gt + pl.dadj_g;
  L.xs = pl.dadj_xs;
  L.X1 = L.X + kAdjBatch * L.xs;
  L.Y = L.X1 + kAdjBatch * L.xs;
  L.Yd = L.Y + kAdjBatch * 16;
  L.B = L.Yd + kAdjBatch * 16;
  L.Bd = L.B + kAdjBatch * RM;
  L.S = L.Bd + kAdjBatch * RM;
  L.Acc = (L.S + kAdjBatch + 3) & ~3;
  return L;
}

__device__ __forceinline__ void dadj_stage_G(const DevPlan& pl, float* dstbase, int rl, int c0, int cw,
                                             const float* __restrict__ G, int nc) {
  for (int p = 0; p < pl.P; ++p) {
    const DevPath& q = pl.path[p];
    const int w = min(cw, q.c_in - c0);
    if (w <= 0) continue;
    const int n3 = 2 * q.l3 + 1, Kb = pl.Kb[q.i3];
    const int w4 = w >> 2;
    const float* src = G + size_t(nc) * pl.a_pref[q.i3] + size_t(rl) * n3 * Kb + q.koff + c0;
    float* dst = dstbase + q.adj_goff * cw;
    const int total = pl.R * n3 * w4;
    for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
      const int row = idx / w4, c = idx - row * w4;
      const int k = row / n3, m3 = row - k * n3;
      cp_async16(dst + row * cw + 4 * c, src + size_t(m3) * Kb + size_t(k) * q.c_in + 4 * c);
    }
  }
}

__device__ __forceinline__ void dadj_stage_X(const DevPlan& pl, float* dst, int xs, const int* scol, int nb, int c0,
                                             int cw, const float* __restrict__ x) {
  int xo = 0;
  for (int i = 0; i < pl.n_in; ++i) {
    const int w = min(cw, pl.in_mul[i] - c0);
    if (w <= 0) continue;
    const int n1 = 2 * pl.in_l[i] + 1, len = w * n1;
    const int so = pl.in_off[i] + c0 * n1;
    for (int idx = threadIdx.x; idx < nb * len; idx += blockDim.x) {
      const int j = idx / len, o = idx - j * len;
      cp_async4(dst + j * xs + xo + o, x + size_t(scol[j]) * pl.dim_in + so + o);
    }
    xo += len;
  }
}

template <int L1, int L2, int L3, int RM>
__device__ __forceinline__ void dadj_tile(const float* xr, const float* x1r, const float* Gp, const float* Gtp,
                                          int cw, int w, const float* Mv, const float* Mdv, const float* bv,
                                          const float* bdv, float* wY, float* hY, float* wb, float* hb) {
  using TR = Tri<L1, L2, L3>;
  constexpr int N1 = TR::N1, N2 = TR::N2, N3 = TR::N3;
  for (int u = 0; u < w; ++u) {
    float xv[N1], x1[N1], T0[N3], T12[N3], dG[N3], dX[N3];
#pragma unroll
    for (int i = 0; i < N1; ++i) {
      xv[i] = xr[u * N1 + i];
      x1[i] = x1r ? x1r[u * N1 + i] : 0.f;
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
        const float g = Gp[(k * N3 + i) * cw + u];
        const float gt = Gtp ? Gtp[(k * N3 + i) * cw + u] : 0.f;
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
      wY[i] += t1[i] + t2[i];
      hY[i] += t3[i];
    }
  }
}

template <int L1, int L2, int L3, int RM>
__device__ __forceinline__ void dadj_path(const DevPlan& pl, const DevPath* pa, const DadjLay& L, float* sm, int rl,
                                          int nb, const float* __restrict__ G, const float* __restrict__ Gt, int nc,
                                          const float* __restrict__ x, const float* __restrict__ ggx) {
  using TR = Tri<L1, L2, L3>;
  constexpr int N2 = TR::N2, NMZ = TR::NMZ;
  const int lane = lane_id();
  const bool live = pa && lane < nb;
  float Mv[NMZ > 0 ? NMZ : 1], Mdv[NMZ > 0 ? NMZ : 1], bv[RM], bdv[RM], wY[N2], hY[N2], wb[RM], hb[RM];
#pragma unroll
  for (int i = 0; i < N2; ++i) wY[i] = hY[i] = 0.f;
#pragma unroll
  for (int k = 0; k < RM; ++k) wb[k] = hb[k] = bv[k] = bdv[k] = 0.f;
  if (live) {
    coupling_row<L1, L2, L3>(sm + L.Y + lane * 16 + L2 * L2, Mv);
    coupling_row<L1, L2, L3>(sm + L.Yd + lane * 16 + L2 * L2, Mdv);
#pragma unroll
    for (int k = 0; k < RM; ++k) {
      bv[k] = sm[L.B + lane * RM + k];
      bdv[k] = sm[L.Bd + lane * RM + k];
    }
  }
  const int cw = pl.dadj_cw;
  const int ntile = (pl.max_c_in + cw - 1) / cw;
  const int* scol = reinterpret_cast<const int*>(sm + L.S);
  for (int t = 0; t < ntile; ++t) {
    const int c0 = t * cw;
    dadj_stage_G(pl, sm + L.G, rl, c0, cw, G, nc);
    if (Gt) dadj_stage_G(pl, sm + L.Gt, rl, c0, cw, Gt, nc);
    dadj_stage_X(pl, sm + L.X, L.xs, scol, nb, c0, cw, x);
    if (ggx) dadj_stage_X(pl, sm + L.X1, L.xs, scol, nb, c0, cw, ggx);
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
    if (live && c0 < pa->c_in) {
      const int xo = adj_xoff(pl, pa->i1, c0, cw);
      dadj_tile<L1, L2, L3, RM>(sm + L.X + lane * L.xs + xo, ggx ? sm + L.X1 + lane * L.xs + xo : nullptr,
                                sm + L.G + pa->adj_goff * cw, Gt ? sm + L.Gt + pa->adj_goff * cw : nullptr, cw,
                                min(cw, pa->c_in - c0), Mv, Mdv, bv, bdv, wY, hY, wb, hb);
    }
    __syncthreads();
  }
  if (live) {
    float* acc = sm + L.Acc + pa->dadj_acc + lane * (2 * N2 + 2 * RM);
#pragma unroll
    for (int i = 0; i < N2; ++i) {
      acc[i] = wY[i];
      acc[N2 + i] = hY[i];
    }
#pragma unroll
    for (int k = 0; k < RM; ++k) {
      acc[2 * N2 + k] = wb[k];
      acc[2 * N2 + RM + k] = hb[k];
    }
  }
}

// grid: receivers in chunk; block: 32 * pl.fz_warps
template <int RM>
__global__ void __launch_bounds__(32 * kFusedMaxWarps, 1)
    k_dadj_stream(const __grid_constant__ DevPlan pl, int r0, int nc, const int* __restrict__ rowptr,
                  const int* __restrict__ col, const float* __restrict__ vec, const float* __restrict__ ggv,
                  const float* __restrict__ x, const float* __restrict__ ggx, const float* __restrict__ G,
                  const float* __restrict__ Gt, float* __restrict__ dvec) {
  extern __shared__ __align__(16) float sm[];
  const DadjLay L = dadj_layout(pl, RM);
  const int warp = threadIdx.x >> 5, lane = lane_id(), nw = blockDim.x >> 5;
  const int rl = blockIdx.x, r = r0 + rl;
  const int e0 = rowptr[r], e1 = rowptr[r + 1];
  for (int eb = e0; eb < e1; eb += kAdjBatch) {
    const int nb = min(kAdjBatch, e1 - eb);
    if (warp == 0 && lane < nb) {
      const int e = eb + lane;
      using D1 = Dual<float, 1>;
      float u[3] = {0.f, 0.f, 0.f};
      if (ggv) load3(ggv, e, u);
      D1 vx(vec[3 * e]), vy(vec[3 * e + 1]), vz(vec[3 * e + 2]);
      vx.d[0] = u[0];
      vy.d[0] = u[1];
      vz.d[0] = u[2];
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
    __syncthreads();
    for (int p0 = 0; p0 < pl.P; p0 += nw) {
      const int p = p0 + warp;
      const DevPath* pa = p < pl.P ? &pl.path[p] : nullptr;
      const int tid = pa ? triple_id(pa->l1, pa->l2, pa->l3) : -1;
      switch (tid) {
#define TPC_CASE(a, b, c)                                                       \
  case triple_id(a, b, c):                                                      \
    dadj_path<a, b, c, RM>(pl, pa, L, sm, rl, nb, G, Gt, nc, x, ggx);           \
    break;
        TPC_FOR_EACH_TRIPLE(TPC_CASE)
#undef TPC_CASE
        default: dadj_path<0, 0, 0, RM>(pl, nullptr, L, sm, rl, nb, G, Gt, nc, x, ggx); break;
      }
    }
    __syncthreads();
    if (warp == 0 && lane < nb) {
      const int e = eb + lane;
      float wY[16], hY[16], wb[RM], hb[RM];
#pragma unroll
      for (int m = 0; m < 16; ++m) wY[m] = hY[m] = 0.f;
#pragma unroll
      for (int k = 0; k < RM; ++k) wb[k] = hb[k] = 0.f;
      for (int p = 0; p < pl.P; ++p) {
        const DevPath& pa = pl.path[p];
        const int N2 = 2 * pa.l2 + 1, o = pa.l2 * pa.l2;
        const float* acc = sm + L.Acc + pa.dadj_acc + lane * (2 * N2 + 2 * RM);
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
