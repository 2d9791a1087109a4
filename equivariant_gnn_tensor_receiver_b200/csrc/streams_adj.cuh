// Receiver adjoint stream with lane = edge.
//
// The per-edge adjoints of the first-order backward,
//     db_ek = sum_{p,u,m3} G[r,k,p,u,m3] T_e[p,u,m3],    T_e = M_e x_s
//     dY_e  = sum_p sum_u C_p(x_s[u], sum_k b_ek G[r,k,p,u])
// are contractions over channels, so each lane owns one edge and accumulates
// its dY_e, db_e in registers: there is no cross-lane reduction.  G_r = Theta^T g_r
// (one channel tile of the receiver's state, all paths) is staged in shared
// memory and read by all lanes at the same address (broadcast float4 over four
// channels); the edge's coupling matrix M_e and radial basis b_e stay in its
// lane's registers.  The gathered rows x_s of a batch of 32 edges are staged
// with an odd row stride, so 32 lanes reading one offset of 32 rows hit 32
// banks.  One warp per path; paths beyond the warp count run in passes.
// d_vec = J_Y^T dY + J_b^T db with forward-mode dual numbers.
//
// Backward of the streaming schedule ("Sobek", arXiv 2607.18074, abstract: the
// reassociation extends through the backward).
#pragma once

#include "streams_v2.cuh"

namespace tpc {

constexpr int kAdjBatch = 32;

struct AdjLay {
  int G, X, Y, B, S, Acc;
  int xs;  // staged row stride (odd)
};

__device__ __forceinline__ AdjLay adj_layout(const DevPlan& pl, int RM) {
  AdjLay L;
  L.G = 0;
  L.X = L.G + pl.adj_g;
  L.xs = pl.adj_xs;
  L.Y = L.X + kAdjBatch * L.xs;
  L.B = L.Y + kAdjBatch * 16;
  L.S = L.B + kAdjBatch * RM;
  L.Acc = (L.S + kAdjBatch + 3) & ~3;
  return L;
}

// offset of input block i1 inside a staged row for the channel tile starting at c0
__device__ __forceinline__ int adj_xoff(const DevPlan& pl, int i1, int c0, int cw) {
  int o = 0;
  for (int i = 0; i < i1; ++i) o += max(0, min(cw, pl.in_mul[i] - c0)) * (2 * pl.in_l[i] + 1);
  return o;
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}

// Stage channel tile [c0, c0+cw) of G_r (all paths, layout [p][k][m3][c]) and of
// the batch's gathered rows x_s.  All threads; returns after the copies landed
// and a barrier.
template <int RM>
__device__ __forceinline__ void adj_stage_tile(const DevPlan& pl, const AdjLay& L, float* sm, int rl, int nb, int c0,
                                               int cw, const float* __restrict__ G, int nc,
                                               const float* __restrict__ x) {
  const int nt = blockDim.x;
  for (int p = 0; p < pl.P; ++p) {
    const DevPath& q = pl.path[p];
    const int w = min(cw, q.c_in - c0);
    if (w <= 0) continue;
    const int n3 = 2 * q.l3 + 1, Kb = pl.Kb[q.i3];
    const int w4 = w >> 2;
    const float* src = G + size_t(nc) * pl.a_pref[q.i3] + size_t(rl) * n3 * Kb + q.koff + c0;
    float* dst = sm + L.G + q.adj_goff * cw;
    const int total = pl.R * n3 * w4;
    for (int idx = threadIdx.x; idx < total; idx += nt) {
      const int row = idx / w4, c = idx - row * w4;  // row = k * n3 + m3
      const int k = row / n3, m3 = row - k * n3;
      cp_async16(dst + row * cw + 4 * c, src + size_t(m3) * Kb + size_t(k) * q.c_in + 4 * c);
    }
  }
  const int* scol = reinterpret_cast<const int*>(sm + L.S);
  int xo = 0;
  for (int i = 0; i < pl.n_in; ++i) {
    const int w = min(cw, pl.in_mul[i] - c0);
    if (w <= 0) continue;
    const int n1 = 2 * pl.in_l[i] + 1, len = w * n1;
    const int so = pl.in_off[i] + c0 * n1;
    for (int idx = threadIdx.x; idx < nb * len; idx += nt) {
      const int j = idx / len, o = idx - j * len;
      cp_async4(sm + L.X + j * L.xs + xo + o, x + size_t(scol[j]) * pl.dim_in + so + o);
    }
    xo += len;
  }
  cp_async_commit();
  cp_async_wait_all();
  __syncthreads();
}

// channels handled per inner step: as many as keep the per-lane temporaries small
template <int N1, int N3>
struct AdjQ {
  static constexpr int value = (N1 + 2 * N3) <= 9 ? 4 : ((N1 + 2 * N3) <= 15 ? 2 : 1);
};

template <int Q>
__device__ __forceinline__ void ldq(const float* p, float* v) {
  if constexpr (Q == 4) {
    const float4 t = *reinterpret_cast<const float4*>(p);
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
  } else if constexpr (Q == 2) {
    const float2 t = *reinterpret_cast<const float2*>(p);
    v[0] = t.x; v[1] = t.y;
  } else {
    v[0] = *p;
  }
}

// one path, one channel tile: accumulate into this lane's dY, db
template <int L1, int L2, int L3, int RM>
__device__ __forceinline__ void adj_tile(const float* xr, const float* Gp, int cw, int w, const float* Mv,
                                         const float* bv, float* dY, float* db) {
  using TR = Tri<L1, L2, L3>;
  constexpr int N1 = TR::N1, N2 = TR::N2, N3 = TR::N3;
  constexpr int Q = AdjQ<N1, N3>::value;
  for (int u = 0; u < w; u += Q) {
    float xv[Q][N1], T[Q][N3], dT[Q][N3];
#pragma unroll
    for (int q = 0; q < Q; ++q) {
#pragma unroll
      for (int i = 0; i < N1; ++i) xv[q][i] = xr[(u + q) * N1 + i];
      apply_M<L1, L2, L3>(Mv, xv[q], T[q]);
#pragma unroll
      for (int i = 0; i < N3; ++i) dT[q][i] = 0.f;
    }
#pragma unroll
    for (int k = 0; k < RM; ++k) {
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < N3; ++i) {
        float g[Q];
        ldq<Q>(Gp + (k * N3 + i) * cw + u, g);
#pragma unroll
        for (int q = 0; q < Q; ++q) {
          dT[q][i] = fmaf(bv[k], g[q], dT[q][i]);
          s = fmaf(g[q], T[q][i], s);
        }
      }
      db[k] += s;
    }
#pragma unroll
    for (int q = 0; q < Q; ++q) {
      float t[N2];
      cg_contract_13<L1, L2, L3>(xv[q], dT[q], t);
#pragma unroll
      for (int i = 0; i < N2; ++i) dY[i] += t[i];
    }
  }
}

// one path over one batch (all channel tiles).  Every warp runs the same
// sequence of staging barriers, whether or not it has a path in this pass.
template <int L1, int L2, int L3, int RM>
__device__ __forceinline__ void adj_path(const DevPlan& pl, const DevPath* pa, const AdjLay& L, float* sm, int rl,
                                         int nb, const float* __restrict__ G, int nc, const float* __restrict__ x) {
  using TR = Tri<L1, L2, L3>;
  constexpr int N2 = TR::N2, NMZ = TR::NMZ;
  const int lane = lane_id();
  const bool live = pa && lane < nb;
  float Mv[NMZ > 0 ? NMZ : 1], bv[RM], dY[N2], db[RM];
#pragma unroll
  for (int i = 0; i < N2; ++i) dY[i] = 0.f;
#pragma unroll
  for (int k = 0; k < RM; ++k) db[k] = bv[k] = 0.f;
  if (live) {
    coupling_row<L1, L2, L3>(sm + L.Y + lane * 16 + L2 * L2, Mv);
#pragma unroll
    for (int k = 0; k < RM; ++k) bv[k] = sm[L.B + lane * RM + k];
  }
  const int cw = pl.adj_cw;
  const int ntile = (pl.max_c_in + cw - 1) / cw;
  for (int t = 0; t < ntile; ++t) {
    const int c0 = t * cw;
    adj_stage_tile<RM>(pl, L, sm, rl, nb, c0, cw, G, nc, x);
    if (live && c0 < pa->c_in) {
      const float* xr = sm + L.X + lane * L.xs + adj_xoff(pl, pa->i1, c0, cw);
      adj_tile<L1, L2, L3, RM>(xr, sm + L.G + pa->adj_goff * cw, cw, min(cw, pa->c_in - c0), Mv, bv, dY, db);
    }
    __syncthreads();
  }
  if (live) {
    float* acc = sm + L.Acc + pa->adj_acc + lane * (N2 + RM);
#pragma unroll
    for (int i = 0; i < N2; ++i) acc[i] = dY[i];
#pragma unroll
    for (int k = 0; k < RM; ++k) acc[N2 + k] = db[k];
  }
}

// grid: receivers in chunk; block: 32 * pl.fz_warps
template <int RM>
__global__ void __launch_bounds__(32 * kFusedMaxWarps, 1)
    k_adj_stream(const __grid_constant__ DevPlan pl, int r0, int nc, const int* __restrict__ rowptr,
                 const int* __restrict__ col, const float* __restrict__ vec, const float* __restrict__ x,
                 const float* __restrict__ G, float* __restrict__ dvec, float* __restrict__ dYout,
                 float* __restrict__ dbout) {
  extern __shared__ __align__(16) float sm[];
  const AdjLay L = adj_layout(pl, RM);
  const int warp = threadIdx.x >> 5, lane = lane_id(), nw = blockDim.x >> 5;
  const int rl = blockIdx.x, r = r0 + rl;
  const int e0 = rowptr[r], e1 = rowptr[r + 1];
  for (int eb = e0; eb < e1; eb += kAdjBatch) {
    const int nb = min(kAdjBatch, e1 - eb);
    if (warp == 0 && lane < nb) {
      const int e = eb + lane;
      float nx, ny, nz, rr;
      unit(vec[3 * e], vec[3 * e + 1], vec[3 * e + 2], nx, ny, nz, rr);
      float* Y = sm + L.Y + lane * 16;
      switch (pl.lsh) {
        case 0: sh_all<0>(nx, ny, nz, Y); break;
        case 1: sh_all<1>(nx, ny, nz, Y); break;
        case 2: sh_all<2>(nx, ny, nz, Y); break;
        default: sh_all<3>(nx, ny, nz, Y); break;
      }
      radial_basis<RM>(pl, rr, sm + L.B + lane * RM);
      reinterpret_cast<int*>(sm + L.S)[lane] = col[e];
    }
    __syncthreads();
    for (int p0 = 0; p0 < pl.P; p0 += nw) {
      const int p = p0 + warp;
      const DevPath* pa = p < pl.P ? &pl.path[p] : nullptr;
      const int tid = pa ? triple_id(pa->l1, pa->l2, pa->l3) : -1;
      switch (tid) {
#define TPC_CASE(a, b, c)                                                    \
  case triple_id(a, b, c):                                                   \
    adj_path<a, b, c, RM>(pl, pa, L, sm, rl, nb, G, nc, x);                  \
    break;
        TPC_FOR_EACH_TRIPLE(TPC_CASE)
#undef TPC_CASE
        default: adj_path<0, 0, 0, RM>(pl, nullptr, L, sm, rl, nb, G, nc, x); break;
      }
    }
    __syncthreads();
    if (warp == 0 && lane < nb) {
      const int e = eb + lane;
      float dY[16], db[RM];
#pragma unroll
      for (int m = 0; m < 16; ++m) dY[m] = 0.f;
#pragma unroll
      for (int k = 0; k < RM; ++k) db[k] = 0.f;
      for (int p = 0; p < pl.P; ++p) {
        const DevPath& pa = pl.path[p];
        const int N2 = 2 * pa.l2 + 1, o = pa.l2 * pa.l2;
        const float* acc = sm + L.Acc + pa.adj_acc + lane * (N2 + RM);
#pragma unroll
        for (int m = 0; m < 16; ++m)
          if (m >= o && m < o + N2) dY[m] += acc[m - o];
#pragma unroll
        for (int k = 0; k < RM; ++k) db[k] += acc[N2 + k];
      }
      if (dvec) {
        const float v[3] = {vec[3 * e], vec[3 * e + 1], vec[3 * e + 2]};
        float o3[3];
        edge_vec_grad<RM>(pl, v, dY, db, o3);
        dvec[3 * e] = o3[0];
        dvec[3 * e + 1] = o3[1];
        dvec[3 * e + 2] = o3[2];
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
