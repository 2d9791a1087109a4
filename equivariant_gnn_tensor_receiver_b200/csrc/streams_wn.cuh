// Warp-per-node edge streams, lane = channel (receiver and sender forms, first
// and second order).
//
// One warp owns one node of the chunk and walks its CSR segment once per path
// and channel tile.  Lane j computes the geometry of edge j of each 32-edge
// batch (unit vector, spherical harmonics of the path's degree l2, radial basis)
// and the edge's compact coupling matrix M[m1][m3] = sum_m2 C[m1,m2,m3] Y[m2];
// both go to the warp's shared slice and are read back by every lane with
// broadcast 16-byte loads.  The neighbours' feature rows are staged by cp.async
// in sub-batches of kWnSub edges, double-buffered, so the gather of the next
// sub-batch overlaps the FFMA work of the current one.  Lane u keeps the node's
// partial state for its CPL channels in registers over the whole segment and
// writes it once: no block barrier, no cross-warp reduction, no atomics.
//
// Forms (streaming schedule of "Sobek", arXiv 2607.18074, abstract: edge-local
// products consumed directly into bounded node-side state):
//   receiver, first order   A[r,k,u,m3]  = sum_e b_ek (M_e x_s[u])[m3]
//   sender,   first order   B[s,k,w,m1]  = sum_e b_ek (M_e^T g_r[w])[m1]
//   receiver, second order  A1 = sum_e b (M x1 + Md x) + bd (M x),  A0 = sum_e b (M x)
//   sender,   second order  B1 = sum_e b (Md^T g) + bd (M^T g),     B0 = sum_e b (M^T g)
// where Md, bd are the derivatives of M_e, b_e along the edge-vector
// perturbation gg_vec_e and x1 = gg_x (terms with a missing input are zero);
// A0 / B0 are computed only by the P1 instantiations (when the caller needs them).
#pragma once

#include "async_copy.cuh"
#include "streams.cuh"
#include "wn_layout.h"

namespace tpc {

// Geometry of edge e for one path: Y of degree L2 and the radial basis (and,
// when DIR, their derivatives along the perturbation ggv_e of the edge vector).
template <int L2, int RM, bool DIR>
__device__ __forceinline__ void wn_geometry(const DevPlan& pl, const float* __restrict__ vec,
                                            const float* __restrict__ ggv, int e, float* Y, float* Yd, float* b,
                                            float* bd) {
  constexpr int N2 = 2 * L2 + 1;
  if constexpr (!DIR) {
    const float vx = vec[3 * e], vy = vec[3 * e + 1], vz = vec[3 * e + 2];
    float nx, ny, nz, r;
    unit(vx, vy, vz, nx, ny, nz, r);
    sh_degree<L2>(nx, ny, nz, Y);
    radial_basis<RM>(pl, r, b);
  } else {
    using D1 = Dual<float, 1>;
    D1 vx(vec[3 * e]), vy(vec[3 * e + 1]), vz(vec[3 * e + 2]);
    if (ggv) {
      vx.d[0] = ggv[3 * e];
      vy.d[0] = ggv[3 * e + 1];
      vz.d[0] = ggv[3 * e + 2];
    }
    D1 nx, ny, nz, r;
    unit(vx, vy, vz, nx, ny, nz, r);
    D1 Yv[N2], bv[RM];
    sh_degree<L2>(nx, ny, nz, Yv);
    radial_basis<RM>(pl, r, bv);
#pragma unroll
    for (int i = 0; i < N2; ++i) {
      Y[i] = Yv[i].v;
      Yd[i] = Yv[i].d[0];
    }
#pragma unroll
    for (int k = 0; k < RM; ++k) {
      b[k] = bv[k].v;
      bd[k] = bv[k].d[0];
    }
  }
}

// compact coupling matrix of one edge, padded with zeros to NMP entries
template <int L1, int L2, int L3, int NMP>
__device__ __forceinline__ void wn_coupling(const float* Y, float* Mrow) {
  constexpr int NMZ = Tri<L1, L2, L3>::NMZ;
  coupling_row<L1, L2, L3>(Y, Mrow);
#pragma unroll
  for (int i = NMZ; i < NMP; ++i) Mrow[i] = 0.f;
}

// (a.x, a.y) = (b.x, b.y) * (t, t) + (a.x, a.y): two FP32 FMAs in one instruction
__device__ __forceinline__ void ffma2_bcast(float2& a, float2 b, float t) { a = __ffma2_rn(b, make_float2(t, t), a); }

// one path, all channel tiles of the warp's node.  The radial state is kept as
// float2 pairs of consecutive radial indices, so the outer products b (x) T run
// as paired FMAs; shared-memory strides are the path's own compile-time widths.
template <int L1, int L2, int L3, int RM, int CPL, bool RECV, bool DBL, bool P1, bool ADD>
__device__ __forceinline__ void wn_chan_path(const DevPlan& pl, const DevPath& q, const WnLay& L, float* ws, int nl,
                                             int nc, int a0, int a1, const int* __restrict__ nbr,
                                             const int* __restrict__ perm, const float* __restrict__ vec,
                                             const float* __restrict__ ggv, const float* __restrict__ src,
                                             const float* __restrict__ src1, float* __restrict__ out,
                                             float* __restrict__ out0) {
  using TR = Tri<L1, L2, L3>;
  constexpr int N2 = TR::N2, NMZ = TR::NMZ, NMP = (NMZ + 3) & ~3;
  constexpr int NI = RECV ? TR::N1 : TR::N3;  // staged floats per channel
  constexpr int NO = RECV ? TR::N3 : TR::N1;  // state floats per channel and radial index
  constexpr int NPART = P1 ? 2 : 1;           // second order: A0 / B0 wanted
  constexpr int NK2 = RM / 2;                 // radial pairs
  constexpr int NACC = NPART * CPL * NK2 * NO;
  constexpr int XS = (32 * CPL * NI + 3) & ~3;  // staged row stride of this path (<= L.xs)
  constexpr int BUF = kWnSub * XS;
  const int lane = lane_id();
  const int c = RECV ? q.c_in : q.c_out;
  const int dim = RECV ? pl.dim_in : pl.dim_out;
  const int off = RECV ? q.in_off : q.out_off;
  const int ne = a1 - a0;
  const int nsb = (ne + kWnSub - 1) / kWnSub;
  const bool two = DBL && RECV && src1 != nullptr;
  float* sM = ws + L.M;
  float* sB = ws + L.B;
  float* sBd = ws + L.Bd;
  float* sX = ws + L.X;
  float* sX1 = ws + L.X1;

  for (int c0 = 0; c0 < c; c0 += 32 * CPL) {
    const int w = min(32 * CPL, c - c0);
    const int len = w * NI;
    const bool v4 = ((dim | off | len) & 3) == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0 &&
                    (reinterpret_cast<uintptr_t>(src1) & 15) == 0;
    const float* srcc = src + size_t(off) + size_t(c0) * NI;
    const float* src1c = two ? src1 + size_t(off) + size_t(c0) * NI : nullptr;
    // stage the rows of sub-batch sb into buffer sb & 1 (one commit group per call site)
    auto stage = [&](int sb) {
      const int j0 = sb * kWnSub, nb = min(kWnSub, ne - j0);
      float* X = sX + (sb & 1) * BUF;
      float* X1 = sX1 + (sb & 1) * BUF;
      const int* nb_idx = nbr + a0 + j0;
      for (int j = 0; j < nb; ++j) {
        const size_t row = size_t(nb_idx[j]) * dim;
        const float* rs = srcc + row;
        float* xd = X + j * XS;
        if (v4) {
          for (int o = 4 * lane; o < len; o += 128) {
            ac_copy16(xd + o, rs + o);
            if (two) ac_copy16(X1 + j * XS + o, src1c + row + o);
          }
        } else {
          for (int o = lane; o < len; o += 32) {
            ac_copy4(xd + o, rs + o);
            if (two) ac_copy4(X1 + j * XS + o, src1c + row + o);
          }
        }
      }
    };

    float2 acc[NACC];
#pragma unroll
    for (int i = 0; i < NACC; ++i) acc[i] = make_float2(0.f, 0.f);

    if (nsb > 0) stage(0);
    ac_commit();
    for (int sb = 0; sb < nsb; ++sb) {
      const int j0 = sb * kWnSub;
      if ((j0 & 31) == 0) {
        // geometry and coupling matrices of the next 32 edges, lane = edge
        __syncwarp();
        const int j = j0 + lane;
        if (j < ne) {
          const int e = RECV ? a0 + j : perm[a0 + j];
          float Y[N2], Yd[N2], b[RM], bd[RM], Mrow[NMP];
          wn_geometry<L2, RM, DBL>(pl, vec, ggv, e, Y, Yd, b, bd);
          wn_coupling<L1, L2, L3, NMP>(Y, Mrow);
          sts_vec<RM>(sB + lane * RM, b);
          if constexpr (!DBL) {
            sts_vec<NMP>(sM + lane * NMP, Mrow);
          } else {
            // (M, Md) side by side: [edge][mi][2] over the M and Md regions
            float Mdrow[NMP], MM[2 * NMP];
            wn_coupling<L1, L2, L3, NMP>(Yd, Mdrow);
#pragma unroll
            for (int i = 0; i < NMP; ++i) {
              MM[2 * i] = Mrow[i];
              MM[2 * i + 1] = Mdrow[i];
            }
            sts_vec<2 * NMP>(sM + lane * 2 * NMP, MM);
            sts_vec<RM>(sBd + lane * RM, bd);
          }
        }
        __syncwarp();
      }
      if (sb + 1 < nsb) stage(sb + 1);
      ac_commit();
      ac_wait<1>();
      __syncwarp();
      const int nb = min(kWnSub, ne - j0);
      const float* Mp = sM + (j0 & 31) * (DBL ? 2 * NMP : NMP);
      const float* Bp = sB + (j0 & 31) * RM;
      const float* Bdp = sBd + (j0 & 31) * RM;
      const float* Xp = sX + (sb & 1) * BUF + lane * NI;
      const float* X1p = sX1 + (sb & 1) * BUF + lane * NI;
      for (int jj = 0; jj < nb; ++jj, Mp += (DBL ? 2 * NMP : NMP), Bp += RM, Bdp += RM, Xp += XS, X1p += XS) {
        float Mv[DBL ? 1 : NMP];
        float2 MM[DBL ? NMP : 1];  // second order: (M, Md) pairs
        float2 b2[NK2];
        if constexpr (!DBL) lds_vec<NMP>(Mp, Mv);
        else lds_f2<NMP>(Mp, MM);
        lds_f2<NK2>(Bp, b2);
        float2 bd2[DBL ? NK2 : 1];
        if constexpr (DBL) lds_f2<NK2>(Bdp, bd2);
#pragma unroll
        for (int h = 0; h < CPL; ++h) {
          float xv[NI];
#pragma unroll
          for (int i = 0; i < NI; ++i) xv[i] = Xp[32 * NI * h + i];
          float2* a = acc + h * NK2 * NO;                 // part 0
          float2* a1 = acc + (P1 ? (CPL + h) * NK2 * NO : 0);  // part 1 (A0 / B0)
          if constexpr (!DBL) {
            float T[NO];
            if constexpr (RECV) apply_M<L1, L2, L3>(Mv, xv, T);
            else apply_Mt<L1, L2, L3>(Mv, xv, T);
#pragma unroll
            for (int kp = 0; kp < NK2; ++kp)
#pragma unroll
              for (int i = 0; i < NO; ++i) ffma2_bcast(a[kp * NO + i], b2[kp], T[i]);
          } else if constexpr (RECV) {
            float x1v[NI], T[NO], T1[NO];
            float2 TT[NO];  // (M x, Md x)
#pragma unroll
            for (int i = 0; i < NI; ++i) x1v[i] = two ? X1p[i] : 0.f;
            apply_M2<L1, L2, L3>(MM, xv, TT);
            apply_M_first<L1, L2, L3>(MM, x1v, T1);
#pragma unroll
            for (int i = 0; i < NO; ++i) {
              T[i] = TT[i].x;
              T1[i] += TT[i].y;
            }
#pragma unroll
            for (int kp = 0; kp < NK2; ++kp)
#pragma unroll
              for (int i = 0; i < NO; ++i) {
                ffma2_bcast(a[kp * NO + i], bd2[kp], T[i]);
                ffma2_bcast(a[kp * NO + i], b2[kp], T1[i]);
                if constexpr (P1) ffma2_bcast(a1[kp * NO + i], b2[kp], T[i]);
              }
          } else {
            float2 UU[NO];  // (M^T g, Md^T g)
            apply_Mt2<L1, L2, L3>(MM, xv, UU);
            float U[NO], U1[NO];
#pragma unroll
            for (int i = 0; i < NO; ++i) {
              U[i] = UU[i].x;
              U1[i] = UU[i].y;
            }
#pragma unroll
            for (int kp = 0; kp < NK2; ++kp)
#pragma unroll
              for (int i = 0; i < NO; ++i) {
                ffma2_bcast(a[kp * NO + i], bd2[kp], U[i]);
                ffma2_bcast(a[kp * NO + i], b2[kp], U1[i]);
                if constexpr (P1) ffma2_bcast(a1[kp * NO + i], b2[kp], U[i]);
              }
          }
        }
      }
      __syncwarp();
    }

    // node state rows: A block i3 (B block i1), row nl * NO + i, column koff + k * c + channel
    const int Kq = RECV ? pl.Kb[q.i3] : pl.Kx[q.i1];
    const int64_t pref = RECV ? pl.a_pref[q.i3] : pl.b_pref[q.i1];
    const size_t base = size_t(nc) * pref + size_t(nl) * NO * Kq + (RECV ? q.koff : q.kxoff) + c0;
#pragma unroll
    for (int part = 0; part < NPART; ++part) {
      float* dst = part == 0 ? out : out0;
#pragma unroll
      for (int h = 0; h < CPL; ++h) {
        const int ch = lane + 32 * h;
        if (ch >= w) continue;
#pragma unroll
        for (int kp = 0; kp < NK2; ++kp)
#pragma unroll
          for (int i = 0; i < NO; ++i) {
            const float2 v = acc[((part * CPL + h) * NK2 + kp) * NO + i];
            float* d = dst + base + size_t(i) * Kq + ch;
            if constexpr (ADD) {  // a further piece of a long segment: add onto the first piece's rows
              if (2 * kp < pl.R) atomicAdd(d + size_t(2 * kp) * c, v.x);
              if (2 * kp + 1 < pl.R) atomicAdd(d + size_t(2 * kp + 1) * c, v.y);
            } else {
              if (2 * kp < pl.R) d[size_t(2 * kp) * c] = v.x;
              if (2 * kp + 1 < pl.R) d[size_t(2 * kp + 1) * c] = v.y;
            }
          }
      }
    }
  }
}

// Two launches per call.  First (EXTRA = false): a path-major grid of
// P * ceil(nc / kWnWarps) CTAs, CTA b running path b / nblk for nodes
// (b % nblk) * kWnWarps + warp; each warp takes its node's whole segment, or the
// first `seg` edges of a longer one.  CTAs are dispatched roughly in index
// order, so the resident warps share one or two path bodies in the instruction
// caches.  Second (EXTRA = true): a persistent grid whose warps claim the
// further pieces of long segments, path-major, from *counter (list `extra`,
// see graph.cuh); it ends at once when no segment is split.  Every node's
// first piece stores its state rows (first launch); the further pieces add onto
// them (second launch, which starts after the first has finished).
// RECV: ptr = rowptr, nbr = col (edge id = CSR position); else ptr = s_rowptr,
// nbr = s_recv, perm = sender-sorted position -> edge id.
// CTAs per SM the register budget is sized for: the second-order forms with
// l = 3 features hold 2 by shared memory (their coupling rows and staged rows
// are longer), so they get the registers of 2
template <int LF, bool RECV, bool DBL>
constexpr int wn_min_ctas() {
  return DBL && LF >= 3 ? 2 : (DBL && RECV ? 3 : 4);
}

template <int RM, int LF, int CPL, bool RECV, bool DBL, bool P1, bool EXTRA>
__global__ void __launch_bounds__(32 * kWnWarps, wn_min_ctas<LF, RECV, DBL>())
    k_wn_stream(const __grid_constant__ DevPlan pl, int n0, int nc, const int* __restrict__ ptr,
                const int* __restrict__ nbr, const int* __restrict__ perm, const float* __restrict__ vec,
                const float* __restrict__ ggv, const float* __restrict__ src, const float* __restrict__ src1,
                float* __restrict__ out, float* __restrict__ out0, const int* __restrict__ extra,
                int* __restrict__ counter, int seg) {
  extern __shared__ __align__(16) float sm[];
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const WnLay L = wn_layout_of(RM, CPL, RECV ? pl.n1max : pl.n3max, pl.nmz_max, DBL, DBL && RECV);
  float* ws = sm + warp * L.total;
  int claim = 0, ne = 0, total = 0;
  if constexpr (EXTRA) {
    ne = extra[nc];
    total = pl.P * ne;
    if (total == 0) return;
    // the next piece is claimed while the current one runs (hides the atomic's latency)
    claim = lane == 0 ? atomicAdd(counter, 1) : 0;
  }
  for (;;) {  // first launch: one pass; second launch: the claimed pieces
    int p, nl, k;
    if constexpr (!EXTRA) {
      const int nblk = (nc + kWnWarps - 1) / kWnWarps;
      p = blockIdx.x / nblk;
      nl = (blockIdx.x - p * nblk) * kWnWarps + warp;
      k = 0;
      if (nl >= nc) break;
    } else {
      const int g = __shfl_sync(0xffffffffu, claim, 0);
      if (g >= total) break;
      if (lane == 0) claim = atomicAdd(counter, 1);
      p = g / ne;
      const int u = g - p * ne;
      nl = extra_owner(extra, nc, u);
      k = 1 + (u - extra[nl]);
    }
    const int s0 = ptr[n0 + nl], s1 = ptr[n0 + nl + 1];
    const int a0 = s0 + k * seg, a1 = min(s1, a0 + seg);
    const DevPath& q = pl.path[p];
    switch (triple_id(q.l1, q.l2, q.l3)) {
#define TPC_CASE(a, b, c)                                                                                        \
  case triple_id(a, b, c):                                                                                       \
    if constexpr (a <= LF && c <= LF)                                                                            \
      wn_chan_path<a, b, c, RM, CPL, RECV, DBL, P1, EXTRA>(pl, q, L, ws, nl, nc, a0, a1, nbr, perm, vec, ggv, src, \
                                                           src1, out, out0);                                     \
    break;
      TPC_FOR_EACH_TRIPLE(TPC_CASE)
#undef TPC_CASE
      default: break;
    }
    if constexpr (!EXTRA) break;
  }
}

}  // namespace tpc
