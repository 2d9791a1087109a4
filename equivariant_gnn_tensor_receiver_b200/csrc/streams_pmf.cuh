// Path-major node streams (lane = channel): forward receiver stream, backward
// sender stream and their double-backward forms.
//
// One CTA per node; all warps work on the same path at the same time (paths are
// iterated uniformly, one hot body in the instruction cache).  The warps split
// the node's edges round-robin, so their work is balanced; lane = channel and
// every lane accumulates its (k, m) state over its warp's edges in registers.
// At the end of a path the warps' partial states are summed through shared
// memory and the path's node-side state is written once, coalesced.
//
//   forward  A[r, k, p, u, m3] = sum_{e->r} b_ek sum_m1 M_e[m1][m3] x[s_e, u, m1]
//   sender   B[s, k, p, w, m1] = sum_{s->e} b_ek sum_m3 M_e[m1][m3] g[r_e, w, m3]
//   double backward (forward form):  A1 = sum b (M gg_x + Mdot x) + bdot M x,  A0 = sum b M x
//   double backward (sender form):   B1 = sum b Mdot^T g + bdot M^T g,         B0 = sum b M^T g
//
// Streaming schedule of "Sobek" (arXiv 2607.18074, abstract): edge-local
// products are consumed directly into bounded node-side state.
#pragma once

#include "pf_layout.h"
#include "pm_layout.h"
#include "streams_dbl.cuh"
#include "streams_v2.cuh"

namespace tpc {

// geometry of edge slots [j0, j0+n) of the node (slot = position in the node's
// edge list modulo kPfGeoMax): Y, b and, when dir, their derivatives along ggv.
// Thread = edge, all threads of the CTA.
template <int RM>
__device__ __forceinline__ void pf_geometry(const DevPlan& pl, const PfLay& L, float* sm, int jb, int n,
                                            const int* __restrict__ nbr, const int* __restrict__ eid,
                                            const float* __restrict__ vec, const float* __restrict__ ggv, bool dir,
                                            int slot0) {
  for (int t = threadIdx.x; t < n; t += blockDim.x) {
    const int e = eid ? eid[jb + t] : jb + t;
    const int sl = slot0 + t;
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
      sm[L.Y + sl * 16 + m] = Y[m].v;
      sm[L.Yd + sl * 16 + m] = Y[m].d[0];
    }
#pragma unroll
    for (int k = 0; k < RM; ++k) {
      sm[L.B + sl * RM + k] = b[k].v;
      sm[L.Bd + sl * RM + k] = b[k].d[0];
    }
    reinterpret_cast<int*>(sm + L.S)[sl] = nbr[jb + t];
  }
}

// entry mi of the compact coupling matrix for the degree-L2 vector Y
template <int L1, int L2, int L3>
__device__ __forceinline__ float coupling_entry(int mi, const float* Y) {
  using TR = Tri<L1, L2, L3>;
  float out = 0.f;
  sfor<TR::N1>([&](auto I1) {
    sfor<TR::N3>([&](auto I3) {
      constexpr int i1 = decltype(I1)::value, i3 = decltype(I3)::value;
      if constexpr (TR::tab.m[i1][i3]) {
        constexpr int m = TR::tab.mi[i1][i3];
        if (mi == m) {
          float s = 0.f;
          sfor<TR::N2>([&](auto I2) {
            constexpr int i2 = decltype(I2)::value;
            if constexpr (TR::tab.cg[i1][i2][i3]) s = fmaf(TR::template cg<i1, i2, i3>(), Y[i2], s);
          });
          out = s;
        }
      }
    });
  });
  return out;
}

// coupling matrices (and those of the derivative direction) of batch slots
template <int L1, int L2, int L3, bool DBL>
__device__ __forceinline__ void pf_couplings(const PfLay& L, float* sm, int nb, int slot0) {
  constexpr int NMZ = Tri<L1, L2, L3>::NMZ, NMP = (NMZ + 3) & ~3;
  for (int t = threadIdx.x; t < nb * NMZ; t += blockDim.x) {
    const int j = t / NMZ, mi = t - j * NMZ;
    const int sl = slot0 + j;
    sm[L.M + j * NMP + mi] = coupling_entry<L1, L2, L3>(mi, sm + L.Y + sl * 16 + L2 * L2);
    if (DBL) sm[L.Md + j * NMP + mi] = coupling_entry<L1, L2, L3>(mi, sm + L.Yd + sl * 16 + L2 * L2);
  }
}

// stage rows [off, off + len) of src (and src1) for the batch's neighbours
__device__ __forceinline__ void pf_rows(const PfLay& L, float* sm, int nb, int slot0, int dim, int off, int len,
                                        const float* __restrict__ src, const float* __restrict__ src1) {
  const int* snb = reinterpret_cast<const int*>(sm + L.S) + slot0;
  const bool v4 = ((off | len | dim) & 3) == 0;
  if (v4) {
    const int len4 = len >> 2;
    for (int idx = threadIdx.x; idx < nb * len4; idx += blockDim.x) {
      const int j = idx / len4, o = 4 * (idx - j * len4);
      const size_t g = size_t(snb[j]) * dim + off + o;
      cp_async16_ca(sm + L.X + j * L.xs + o, src + g);
      if (src1) cp_async16_ca(sm + L.X1 + j * L.xs + o, src1 + g);
    }
  } else {
    for (int j = 0; j < nb; ++j) {
      const size_t g = size_t(snb[j]) * dim + off;
      for (int o = threadIdx.x; o < len; o += blockDim.x) {
        cp_async4(sm + L.X + j * L.xs + o, src + g + o);
        if (src1) cp_async4(sm + L.X1 + j * L.xs + o, src1 + g + o);
      }
    }
  }
  cp_async_commit();
}

// sum the warps' partial states (NA floats per lane) in rounds of kPfRedChunk
// and hand every summed value to `emit(a, lane, value)`
template <int NA, class Emit>
__device__ __forceinline__ void pf_reduce(const PfLay& L, float* sm, const float* acc, Emit emit) {
  const int warp = threadIdx.x >> 5, lane = lane_id();
  float* red = sm + L.Red;
#pragma unroll
  for (int a0 = 0; a0 < NA; a0 += kPfRedChunk) {
    constexpr int CH = kPfRedChunk;
#pragma unroll
    for (int i = 0; i < CH; ++i)
      if (a0 + i < NA) red[(warp * CH + i) * 32 + lane] = acc[a0 + i < NA ? a0 + i : 0];
    __syncthreads();
    const int na = min(CH, NA - a0);
    for (int idx = threadIdx.x; idx < na * 32; idx += blockDim.x) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kPmWarps; ++w) s += red[w * CH * 32 + idx];
      emit(a0 + idx / 32, idx % 32, s);
    }
    __syncthreads();
  }
}

// Slot of a batch in the geometry cache; batches beyond the cache get the scratch
// slots (and their geometry is recomputed by the caller).
__device__ __forceinline__ int pf_slot(int off, int nb) { return off + nb <= kPfGeoMax ? off : kPfGeoMax; }

// ---------------------------------------------------------------------------
// receiver-form body (forward; double-backward forward form when DBL)
// ---------------------------------------------------------------------------
template <int L1, int L2, int L3, int RM, bool DBL>
__device__ __forceinline__ void pf_recv_path(const DevPlan& pl, const DevPath& q, const PfLay& L, float* sm, int rl,
                                             int e0, int e1, int c0, const int* __restrict__ col,
                                             const float* __restrict__ vec, const float* __restrict__ ggv,
                                             const float* __restrict__ x, const float* __restrict__ x1,
                                             float* __restrict__ A, float* __restrict__ A0) {
  using TR = Tri<L1, L2, L3>;
  constexpr int N1 = TR::N1, N3 = TR::N3, NMZ = TR::NMZ, NMP = (NMZ + 3) & ~3;
  constexpr int NA = (DBL ? 2 : 1) * RM * N3;
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const int u = c0 + lane;
  const bool act = u < q.c_in;
  float acc[NA];
#pragma unroll
  for (int i = 0; i < NA; ++i) acc[i] = 0.f;
  const int w = min(32, q.c_in - c0);
  for (int eb = e0; eb < e1; eb += kPmBatch) {
    const int nb = min(kPmBatch, e1 - eb);
    const int slot = pf_slot(eb - e0, nb);
    if (slot == kPfGeoMax) {
      pf_geometry<RM>(pl, L, sm, eb, nb, col, nullptr, vec, ggv, DBL, slot);
      __syncthreads();
    }
    pf_rows(L, sm, nb, slot, pl.dim_in, q.in_off + c0 * N1, w * N1, x, DBL ? x1 : nullptr);
    pf_couplings<L1, L2, L3, DBL>(L, sm, nb, slot);
    cp_async_wait_all();
    __syncthreads();
    for (int j = warp; j < nb; j += kPmWarps) {
      const float* Mj = sm + L.M + j * NMP;
      const float* bj = sm + L.B + (slot + j) * RM;
      float xv[N1];
#pragma unroll
      for (int i = 0; i < N1; ++i) xv[i] = act ? sm[L.X + j * L.xs + lane * N1 + i] : 0.f;
      float T[N3];
      if constexpr (!DBL) {
        float Mv[NMP], bv[RM];
#pragma unroll
        for (int i = 0; i < NMP / 4; ++i) {
          const float4 t = reinterpret_cast<const float4*>(Mj)[i];
          Mv[4 * i] = t.x; Mv[4 * i + 1] = t.y; Mv[4 * i + 2] = t.z; Mv[4 * i + 3] = t.w;
        }
#pragma unroll
        for (int i = 0; i < RM / 4; ++i) {
          const float4 t = reinterpret_cast<const float4*>(bj)[i];
          bv[4 * i] = t.x; bv[4 * i + 1] = t.y; bv[4 * i + 2] = t.z; bv[4 * i + 3] = t.w;
        }
        apply_M<L1, L2, L3>(Mv, xv, T);
#pragma unroll
        for (int k = 0; k < RM; ++k)
#pragma unroll
          for (int i = 0; i < N3; ++i) acc[k * N3 + i] = fmaf(bv[k], T[i], acc[k * N3 + i]);
      } else {
        const float* bdj = sm + L.Bd + (slot + j) * RM;
        float x1v[N1], T1[N3], T2[N3];
#pragma unroll
        for (int i = 0; i < N1; ++i) x1v[i] = (act && x1) ? sm[L.X1 + j * L.xs + lane * N1 + i] : 0.f;
        apply_M<L1, L2, L3>(Mj, xv, T);
        apply_M<L1, L2, L3>(Mj, x1v, T1);
        apply_M<L1, L2, L3>(sm + L.Md + j * NMP, xv, T2);
#pragma unroll
        for (int k = 0; k < RM; ++k) {
          const float bk = bj[k], bdk = bdj[k];
#pragma unroll
          for (int i = 0; i < N3; ++i) {
            acc[k * N3 + i] = fmaf(bk, T1[i] + T2[i], fmaf(bdk, T[i], acc[k * N3 + i]));
            acc[RM * N3 + k * N3 + i] = fmaf(bk, T[i], acc[RM * N3 + k * N3 + i]);
          }
        }
      }
    }
    __syncthreads();
  }
  // A row (rl, m3), column koff + k * c_in + u
  const int Kb = pl.Kb[q.i3];
  const size_t base = size_t(gridDim.x) * pl.a_pref[q.i3] + size_t(rl) * N3 * Kb + q.koff + c0;
  pf_reduce<NA>(L, sm, acc, [&](int a, int ln, float v) {
    if (ln >= w) return;
    const int part = a / (RM * N3), ki = a % (RM * N3);
    const int k = ki / N3, i = ki % N3;
    if (k >= pl.R) return;
    float* dst = part == 0 ? A : A0;
    dst[base + size_t(i) * Kb + k * q.c_in + ln] = v;
  });
}

// ---------------------------------------------------------------------------
// sender-form body (backward sender stream; double-backward sender form when DBL)
// ---------------------------------------------------------------------------
template <int L1, int L2, int L3, int RM, bool DBL>
__device__ __forceinline__ void pf_send_path(const DevPlan& pl, const DevPath& q, const PfLay& L, float* sm, int sl,
                                             int j0, int j1, int c0, const int* __restrict__ perm,
                                             const int* __restrict__ s_recv, const float* __restrict__ vec,
                                             const float* __restrict__ ggv, const float* __restrict__ g,
                                             float* __restrict__ B, float* __restrict__ B0) {
  using TR = Tri<L1, L2, L3>;
  constexpr int N1 = TR::N1, N3 = TR::N3, NMZ = TR::NMZ, NMP = (NMZ + 3) & ~3;
  constexpr int NA = (DBL ? 2 : 1) * RM * N1;
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const int wch = c0 + lane;
  const bool act = wch < q.c_out;
  float acc[NA];
#pragma unroll
  for (int i = 0; i < NA; ++i) acc[i] = 0.f;
  const int w = min(32, q.c_out - c0);
  for (int jb = j0; jb < j1; jb += kPmBatch) {
    const int nb = min(kPmBatch, j1 - jb);
    const int slot = pf_slot(jb - j0, nb);
    if (slot == kPfGeoMax) {
      pf_geometry<RM>(pl, L, sm, jb, nb, s_recv, perm, vec, ggv, DBL, slot);
      __syncthreads();
    }
    pf_rows(L, sm, nb, slot, pl.dim_out, q.out_off + c0 * N3, w * N3, g, nullptr);
    pf_couplings<L1, L2, L3, DBL>(L, sm, nb, slot);
    cp_async_wait_all();
    __syncthreads();
    for (int j = warp; j < nb; j += kPmWarps) {
      const float* Mj = sm + L.M + j * NMP;
      const float* bj = sm + L.B + (slot + j) * RM;
      float gv[N3];
#pragma unroll
      for (int i = 0; i < N3; ++i) gv[i] = act ? sm[L.X + j * L.xs + lane * N3 + i] : 0.f;
      float U[N1];
      if constexpr (!DBL) {
        float Mv[NMP], bv[RM];
#pragma unroll
        for (int i = 0; i < NMP / 4; ++i) {
          const float4 t = reinterpret_cast<const float4*>(Mj)[i];
          Mv[4 * i] = t.x; Mv[4 * i + 1] = t.y; Mv[4 * i + 2] = t.z; Mv[4 * i + 3] = t.w;
        }
#pragma unroll
        for (int i = 0; i < RM / 4; ++i) {
          const float4 t = reinterpret_cast<const float4*>(bj)[i];
          bv[4 * i] = t.x; bv[4 * i + 1] = t.y; bv[4 * i + 2] = t.z; bv[4 * i + 3] = t.w;
        }
        apply_Mt<L1, L2, L3>(Mv, gv, U);
#pragma unroll
        for (int k = 0; k < RM; ++k)
#pragma unroll
          for (int i = 0; i < N1; ++i) acc[k * N1 + i] = fmaf(bv[k], U[i], acc[k * N1 + i]);
      } else {
        const float* bdj = sm + L.Bd + (slot + j) * RM;
        float U1[N1];
        apply_Mt<L1, L2, L3>(Mj, gv, U);
        apply_Mt<L1, L2, L3>(sm + L.Md + j * NMP, gv, U1);
#pragma unroll
        for (int k = 0; k < RM; ++k) {
          const float bk = bj[k], bdk = bdj[k];
#pragma unroll
          for (int i = 0; i < N1; ++i) {
            acc[k * N1 + i] = fmaf(bk, U1[i], fmaf(bdk, U[i], acc[k * N1 + i]));
            acc[RM * N1 + k * N1 + i] = fmaf(bk, U[i], acc[RM * N1 + k * N1 + i]);
          }
        }
      }
    }
    __syncthreads();
  }
  const int Kx = pl.Kx[q.i1];
  const size_t base = size_t(gridDim.x) * pl.b_pref[q.i1] + size_t(sl) * N1 * Kx + q.kxoff + c0;
  pf_reduce<NA>(L, sm, acc, [&](int a, int ln, float v) {
    if (ln >= w) return;
    const int part = a / (RM * N1), ki = a % (RM * N1);
    const int k = ki / N1, i = ki % N1;
    if (k >= pl.R) return;
    float* dst = part == 0 ? B : B0;
    dst[base + size_t(i) * Kx + k * q.c_out + ln] = v;
  });
}

// grid: nodes in chunk; block: 32 * kPmWarps.  RECV: receiver form (ptr = rowptr,
// nbr = col), else sender form (ptr = s_rowptr, nbr = s_recv, perm).
template <int RM, bool RECV, bool DBL>
__global__ void __launch_bounds__(32 * kPmWarps, DBL ? 1 : 2)
    k_pf_stream(const __grid_constant__ DevPlan pl, int n0, const int* __restrict__ ptr,
                const int* __restrict__ nbr, const int* __restrict__ perm, const float* __restrict__ vec,
                const float* __restrict__ ggv, const float* __restrict__ src, const float* __restrict__ src1,
                float* __restrict__ out, float* __restrict__ out0) {
  extern __shared__ __align__(16) float sm[];
  const PfLay L = pf_layout_of(RM, RECV ? pl.pm_n1max : pl.pm_n3max, pl.pf_nmz_max, DBL);
  const int nl = blockIdx.x, node = n0 + nl;
  const int a0 = ptr[node], a1 = ptr[node + 1];
  // geometry of the node's first kPfGeoMax edges, shared by every path
  pf_geometry<RM>(pl, L, sm, a0, min(a1 - a0, kPfGeoMax), nbr, RECV ? nullptr : perm, vec, ggv, DBL, 0);
  __syncthreads();
  for (int p = 0; p < pl.P; ++p) {
    const DevPath& q = pl.path[p];
    const int cmax = RECV ? q.c_in : q.c_out;
    for (int c0 = 0; c0 < cmax; c0 += 32) {
      switch (triple_id(q.l1, q.l2, q.l3)) {
#define TPC_CASE(a, b, c)                                                                                   \
  case triple_id(a, b, c):                                                                                  \
    if constexpr (RECV)                                                                                     \
      pf_recv_path<a, b, c, RM, DBL>(pl, q, L, sm, nl, a0, a1, c0, nbr, vec, ggv, src, src1, out, out0);    \
    else                                                                                                    \
      pf_send_path<a, b, c, RM, DBL>(pl, q, L, sm, nl, a0, a1, c0, perm, nbr, vec, ggv, src, out, out0);    \
    break;
        TPC_FOR_EACH_TRIPLE(TPC_CASE)
#undef TPC_CASE
        default: break;
      }
    }
  }
}

}  // namespace tpc
