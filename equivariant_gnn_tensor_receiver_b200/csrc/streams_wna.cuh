// Warp-per-node receiver adjoint streams, lane = edge (first and second order).
//
// Second order: a warp takes 32 consecutive edges of the receiver-sorted CSR
// order (one per lane), whichever receivers they belong to, so every lane does
// useful work; first order (lighter per channel, where staging several
// receivers' rows costs more than the idle lanes): up to 32 edges of one
// receiver.  Either way a hub's edges spread over many warps.  The node-side adjoint state
// G = Theta^T g_r (and, for the double backward, Gt = gg_Theta^T g_r) of the
// receivers present is staged by cp.async in chunks of kWnChunk channels as
// [u][k][m3], one slot per receiver, so that the lanes of one receiver read a
// channel's RM x n3 block with broadcast 16-byte loads, while each lane stages
// and reads its own edge's sender row.  All reductions over channels happen in the lane's
// registers; the CG contraction with the per-edge outer-product accumulator Q
// runs once per path rather than once per channel.
//
// First order (e = s -> r):
//     db_ek = sum_{p,u,m3} G[k,p,u,m3] (M_e x_s[u])[m3]
//     dY_e  = sum_p C_p : Q_p,   Q_p[m1][m3] = sum_u x_s[u,m1] (sum_k b_ek G[k,p,u,m3])
//     dvec_e = J_Y^T dY_e + J_b^T db_e
// Second order (Md, bd along gg_vec_e, x1 = gg_x), per channel:
//     dG = sum_k b_k G_k,  dX = sum_k (b_k Gt_k + bd_k G_k),  T0 = M x,  T12 = M x1 + Md x
//     wb_k += G_k.T12 + Gt_k.T0,  hb_k += G_k.T0
//     Qw += x1 (x) dG + x (x) dX,  Qh += x (x) dG
//     d_vec_e = grad_v [wY.Y + hY.Ydot + wb.b + hb.bdot],  wY = C:Qw, hY = C:Qh
// Backward of the streaming schedule ("Sobek", arXiv 2607.18074, abstract).
#pragma once

#include "async_copy.cuh"
#include "streams_dbl.cuh"
#include "wn_layout.h"

namespace tpc {

// ---- one path restricted to the output components m3 in [A3, B3) -------------
// The per-lane state of a path (coupling rows M, Md and the accumulators Q, Qh)
// has one entry per structural nonzero (m1, m3).  Large paths (l = 3 with
// 26-42 nonzeros) run their channel loop in two passes over halves of the m3
// range, each holding only its half of that state: the same arithmetic, half
// the registers.  TriPart compresses the nonzeros of the restricted range.
template <int L1, int L2, int L3, int A3, int B3>
struct TriPart {
  using TR = Tri<L1, L2, L3>;
  static constexpr int N1 = TR::N1, N2 = TR::N2, N3 = TR::N3;
  struct Tab {
    bool m[N1][N3];
    int mi[N1][N3];
    int nmz;
  };
  static constexpr Tab make() {
    Tab t{};
    int c = 0;
    for (int a = 0; a < N1; ++a)
      for (int b = 0; b < N3; ++b) {
        const bool on = TR::tab.m[a][b] && b >= A3 && b < B3;
        t.m[a][b] = on;
        t.mi[a][b] = on ? c++ : -1;
      }
    t.nmz = c;
    return t;
  }
  static constexpr Tab tab = make();
  static constexpr int NMZ = tab.nmz > 0 ? tab.nmz : 1;
};

// Mrow[mi] = sum_m2 C[m1,m2,m3] Y[m2] on the part's nonzeros
template <class TP, int L1, int L2, int L3>
__device__ __forceinline__ void part_coupling_row(const float* Y, float* Mrow) {
  using TR = Tri<L1, L2, L3>;
  sfor<TR::N1>([&](auto I1) {
    sfor<TR::N3>([&](auto I3) {
      constexpr int i1 = decltype(I1)::value, i3 = decltype(I3)::value;
      if constexpr (TP::tab.m[i1][i3]) {
        float s = 0.f;
        sfor<TR::N2>([&](auto I2) {
          constexpr int i2 = decltype(I2)::value;
          if constexpr (TR::tab.cg[i1][i2][i3]) s = fmaf(TR::template cg<i1, i2, i3>(), Y[i2], s);
        });
        constexpr int mi = TP::tab.mi[i1][i3];
        Mrow[mi] = s;
      }
    });
  });
}
// T[m3] = sum_m1 M[m1][m3] x[m1] for the part's m3 (other entries zero)
template <class TP>
__device__ __forceinline__ void part_apply_M(const float* Mv, const float* xv, float* T) {
#pragma unroll
  for (int i3 = 0; i3 < TP::N3; ++i3) T[i3] = 0.f;
  sfor<TP::N1>([&](auto I1) {
    sfor<TP::N3>([&](auto I3) {
      constexpr int i1 = decltype(I1)::value, i3 = decltype(I3)::value;
      if constexpr (TP::tab.m[i1][i3]) {
        constexpr int mi = TP::tab.mi[i1][i3];
        T[i3] = fmaf(Mv[mi], xv[i1], T[i3]);
      }
    });
  });
}
// (T, Td)[m3] = sum_m1 (M, Md)[m1][m3] x[m1], and T1[m3] = sum_m1 M[m1][m3] x1[m1]
template <class TP>
__device__ __forceinline__ void part_apply_M2(const float2* MM, const float* xv, const float* x1v, float2* TT,
                                              float* T1) {
#pragma unroll
  for (int i3 = 0; i3 < TP::N3; ++i3) {
    TT[i3] = make_float2(0.f, 0.f);
    T1[i3] = 0.f;
  }
  sfor<TP::N1>([&](auto I1) {
    sfor<TP::N3>([&](auto I3) {
      constexpr int i1 = decltype(I1)::value, i3 = decltype(I3)::value;
      if constexpr (TP::tab.m[i1][i3]) {
        constexpr int mi = TP::tab.mi[i1][i3];
        TT[i3] = __ffma2_rn(MM[mi], make_float2(xv[i1], xv[i1]), TT[i3]);
        T1[i3] = fmaf(MM[mi].x, x1v[i1], T1[i3]);
      }
    });
  });
}
// Q[mi] += a[m1] c[m3] on the part's nonzeros
template <class TP>
__device__ __forceinline__ void part_outer_Q(const float* a, const float* c, float* Q) {
  sfor<TP::N1>([&](auto I1) {
    sfor<TP::N3>([&](auto I3) {
      constexpr int i1 = decltype(I1)::value, i3 = decltype(I3)::value;
      if constexpr (TP::tab.m[i1][i3]) {
        constexpr int mi = TP::tab.mi[i1][i3];
        Q[mi] = fmaf(a[i1], c[i3], Q[mi]);
      }
    });
  });
}
// out[m2] += sum_{m1, m3 in the part} C[m1,m2,m3] Q[m1][m3]
template <class TP, int L1, int L2, int L3>
__device__ __forceinline__ void part_contract_Q(const float* Q, float* out) {
  using TR = Tri<L1, L2, L3>;
  sfor<TR::N1>([&](auto I1) {
    sfor<TR::N3>([&](auto I3) {
      constexpr int i1 = decltype(I1)::value, i3 = decltype(I3)::value;
      if constexpr (TP::tab.m[i1][i3]) {
        constexpr int mi = TP::tab.mi[i1][i3];
        sfor<TR::N2>([&](auto I2) {
          constexpr int i2 = decltype(I2)::value;
          if constexpr (TR::tab.cg[i1][i2][i3]) out[i2] = fmaf(TR::template cg<i1, i2, i3>(), Q[mi], out[i2]);
        });
      }
    });
  });
}
// float pairs J0 .. J0+NP-1 of a 16-byte aligned shared array: 16-byte reads
// where the pair index is even, 8-byte reads otherwise (J0, NP compile-time)
template <int J0, int NP>
__device__ __forceinline__ void lds_f2_at(const float* base, float2* v) {
  if constexpr (NP > 0) {
    if constexpr ((J0 & 1) == 0 && NP >= 2) {
      const float4 t = lds4(base + 2 * J0);
      v[0] = make_float2(t.x, t.y);
      v[1] = make_float2(t.z, t.w);
      lds_f2_at<J0 + 2, NP - 2>(base, v + 2);
    } else {
      v[0] = *reinterpret_cast<const float2*>(base + 2 * J0);
      lds_f2_at<J0 + 1, NP - 1>(base, v + 1);
    }
  }
}
// floats OFF .. OFF+N-1 of a 16-byte aligned shared array, in the widest reads
// their alignment allows (OFF, N compile-time)
template <int OFF, int N>
__device__ __forceinline__ void lds_run(const float* base, float* v) {
  if constexpr (N > 0) {
    if constexpr ((OFF & 3) == 0 && N >= 4) {
      const float4 t = lds4(base + OFF);
      v[0] = t.x;
      v[1] = t.y;
      v[2] = t.z;
      v[3] = t.w;
      lds_run<OFF + 4, N - 4>(base, v + 4);
    } else if constexpr ((OFF & 1) == 0 && N >= 2) {
      const float2 t = *reinterpret_cast<const float2*>(base + OFF);
      v[0] = t.x;
      v[1] = t.y;
      lds_run<OFF + 2, N - 2>(base, v + 2);
    } else {
      v[0] = base[OFF];
      lds_run<OFF + 1, N - 1>(base, v + 1);
    }
  }
}
// the m3 halves of a path: split when its per-lane state exceeds this many
// nonzeros (second order with l = 3 features: a lower bound, as their x rows
// and coupling rows are longer)
constexpr int kWnaSplitNmz = 24, kWnaSplitNmzL3 = 16;

// Shared G tiles hold radial pairs side by side, [u][k / 2][m3][k & 1], so that a
// 16-byte read yields float2 operands (G_2kp, G_2kp+1) for paired FMAs.
template <int N3>
__host__ __device__ constexpr int g_slot(int k, int m3) {
  return ((k >> 1) * N3 + m3) * 2 + (k & 1);
}

// one path of one 32-edge batch, output components m3 in [A3, B3) (GT: the
// second order has a Gt operand).  rfirst: chunk-local receiver of lane 0's
// edge; the window's receivers are rfirst .. rfirst + nslots - 1 and the lane's
// is rfirst + myslot (myslot < 0: no edge).  db, hb collect over all parts.
template <int L1, int L2, int L3, int RM, bool DBL, bool GT, bool XB, int A3, int B3>
__device__ __forceinline__ void wna_path(const DevPlan& pl, const DevPath& q, const WnaLay& L, float* ws, int rfirst,
                                         int nslots, int myslot, int nc, int nb, int myrow,
                                         const float* __restrict__ x,
                                         const float* __restrict__ x1, const float* __restrict__ G,
                                         const float* __restrict__ Gt, float2* db, float2* hb) {
  using TR = Tri<L1, L2, L3>;
  using TP = TriPart<L1, L2, L3, A3, B3>;
  constexpr int N1 = TR::N1, N2 = TR::N2, N3 = TR::N3, NMZ = TP::NMZ, GW = RM * N3, NK2 = RM / 2;
  constexpr int NH = B3 - A3;  // m3 components of this part
  constexpr int CH = kWnChunk;
  static_assert(CH == 4, "the chunk is one group of four channels");
  static_assert(0 <= A3 && A3 < B3 && B3 <= N3, "m3 part");
  // channels of a chunk unrolled together: the second-order bodies unroll two
  // (a runtime loop over the pairs), which halves their code against four
  // unrolled channels; instruction fetch stalls were 0.7 cycles per issue with
  // four.  Measured second-order adjoint: mace-like layer 2.29 -> 2.22 ms,
  // sweep at degree 25 2.90 -> 2.71 ms, wide layer 27.1 -> 26.4 ms (one
  // channel at a time: 2.38, 2.64, 28.2 ms).
  constexpr int CHU = DBL ? 2 : CH;
  constexpr int NIT = (RM * NH * CH + 31) / 32;  // G elements of the part per lane and chunk (upper bound)
  const int lane = lane_id();
  const float* geo = ws + L.Geo + lane * L.geos;
  // first order: M in Mv; second order: (M, Md) side by side in MM (paired FMAs);
  // accumulators Q (second order: Qw) and Qh
  float Mv[DBL ? 1 : NMZ];
  float2 MM[DBL ? NMZ : 1];
  float2 b2[NK2], bd2[DBL ? NK2 : 1];
  {
    float Y[N2], Mrow[NMZ];
#pragma unroll
    for (int i = 0; i < N2; ++i) Y[i] = geo[L2 * L2 + i];
    part_coupling_row<TP, L1, L2, L3>(Y, DBL ? Mrow : Mv);
#pragma unroll
    for (int kp = 0; kp < NK2; ++kp) b2[kp] = make_float2(geo[16 + 2 * kp], geo[17 + 2 * kp]);
    if constexpr (DBL) {
      float Mdrow[NMZ];
#pragma unroll
      for (int i = 0; i < N2; ++i) Y[i] = geo[16 + RM + L2 * L2 + i];
      part_coupling_row<TP, L1, L2, L3>(Y, Mdrow);
#pragma unroll
      for (int i = 0; i < NMZ; ++i) MM[i] = make_float2(Mrow[i], Mdrow[i]);
#pragma unroll
      for (int kp = 0; kp < NK2; ++kp) bd2[kp] = make_float2(geo[32 + RM + 2 * kp], geo[33 + RM + 2 * kp]);
    }
  }
  float Q[NMZ], Qh[DBL ? NMZ : 1];
#pragma unroll
  for (int i = 0; i < NMZ; ++i) Q[i] = 0.f;
  if constexpr (DBL) {
#pragma unroll
    for (int i = 0; i < NMZ; ++i) Qh[i] = 0.f;
  }

  const int c = q.c_in, R = pl.R;
  const int nch = c / CH;  // channel counts are multiples of four on this path
  const int Kb = pl.Kb[q.i3];
  constexpr bool has_t = DBL && GT;
  const bool has_x1 = DBL && x1 != nullptr;
  // this lane's G elements of a chunk (the part's m3 only): source offset
  // (relative to receiver row and channel u0) and position inside a slot, the
  // same for every chunk
  const int NS = L.ns;
  const size_t rowstride = size_t(N3) * Kb;
  const float* Gp = G + size_t(nc) * pl.a_pref[q.i3] + size_t(rfirst) * rowstride + q.koff;
  const float* Gtp = has_t ? Gt + (Gp - G) : nullptr;
  int gsrc[NIT], gdst[NIT];
#pragma unroll
  for (int it = 0; it < NIT; ++it) {
    const int t = it * 32 + lane;
    const int u = t & (CH - 1), km = t / CH;  // km = k * NH + (m3 - A3)
    const int k = km / NH, m3 = A3 + (km - k * NH);
    gsrc[it] = k < R ? m3 * Kb + k * c + u : -1;
    gdst[it] = u * GW + g_slot<N3>(k, m3);
  }
  int g0 = 0;  // first receiver slot of the group being staged
  auto stage = [&](int ch) {
    const int u0 = ch * CH;
    const int ns = min(NS, nslots - g0);
    for (int sl = 0; sl < ns; ++sl) {
      float* sG = ws + L.G + (ch & 1) * L.gbuf + sl * L.gslot;
      float* sGt = ws + L.Gt + (ch & 1) * L.gbuf + sl * L.gslot;
      const size_t ro = size_t(g0 + sl) * rowstride + u0;
#pragma unroll
      for (int it = 0; it < NIT; ++it) {
        if (gsrc[it] >= 0) {
          ac_copy4(sG + gdst[it], Gp + ro + gsrc[it]);
          if constexpr (has_t) ac_copy4(sGt + gdst[it], Gtp + ro + gsrc[it]);
        }
      }
    }
    // the batch's rows, N1 16-byte pieces each, copied by the whole warp (coalesced)
    float* sX = ws + L.X + (ch & 1) * L.xbuf;
    float* sX1 = ws + L.X1 + (ch & 1) * L.xbuf;
    const size_t cofs = size_t(q.in_off) + size_t(u0) * N1;
#pragma unroll
    for (int it = 0; it < N1; ++it) {
      const int qd = it * 32 + lane;
      const int j = qd / N1, v = qd - j * N1;
      const int rj = __shfl_sync(0xffffffffu, myrow, j);
      if (j < nb) {
        const size_t src = size_t(rj) * pl.dim_in + cofs + 4 * v;
        ac_copy16(sX + j * L.xs + 4 * v, x + src);
        if (has_x1) ac_copy16(sX1 + j * L.xs + 4 * v, x1 + src);
      }
    }
  };

  // receivers in groups of NS slots (one group unless the window spans more
  // than NS receivers); a lane whose receiver is not in the group adds nothing
  // (its x rows read as zero)
  for (g0 = 0; g0 < nslots; g0 += NS) {
  const bool active = myslot >= g0 && myslot < g0 + NS;
  if (nch > 0) stage(0);
  ac_commit();
  for (int ch = 0; ch < nch; ++ch) {
    if (ch + 1 < nch) stage(ch + 1);
    ac_commit();
    ac_wait<1>();
    __syncwarp();
    // a lane whose receiver is not in this group reads slot 0 and the zero x row
    const int sl = active ? myslot - g0 : 0;  // lanes without an edge (myslot < 0) read slot 0 too
    const float* sG = ws + L.G + (ch & 1) * L.gbuf + sl * L.gslot;
    const float* sGt = ws + L.Gt + (ch & 1) * L.gbuf + sl * L.gslot;
    // the lane's rows of the four channels: all at once in N1 16-byte reads, or
    // in kernels with l = 3 features channel by channel (one channel's x, x1
    // live at a time)
    constexpr bool XBULK = XB;
    // (first order: one group, every lane with an edge is in it)
    const bool xz = DBL && !active;
    const float* sXl = xz ? ws + L.XZ : ws + L.X + (ch & 1) * L.xbuf + lane * L.xs;
    const float* sX1l = xz ? ws + L.XZ : ws + L.X1 + (ch & 1) * L.xbuf + lane * L.xs;
    constexpr bool XB4 = XBULK && CHU == CH;  // bulk x loads need the four channels unrolled
    float xg[XB4 ? CH * N1 : 1], x1g[XB4 && DBL ? CH * N1 : 1];
    if constexpr (XB4) {
      lds_vec<CH * N1>(sXl, xg);
      if constexpr (DBL) lds_vec<CH * N1>(sX1l, x1g);
    }
    // one channel t of the chunk (compile-time when the whole chunk is unrolled)
    auto chan = [&](auto TI, int tg) {
      constexpr int ti = decltype(TI)::value;
      const int t = CHU == CH ? ti : tg + ti;
      float xv[N1];
      if constexpr (CHU < CH) {
#pragma unroll
        for (int i = 0; i < N1; ++i) xv[i] = sXl[t * N1 + i];
      } else if constexpr (XB4) {
#pragma unroll
        for (int i = 0; i < N1; ++i) xv[i] = xg[ti * N1 + i];
      } else {
        lds_run<ti * N1, N1>(sXl, xv);
      }
      if constexpr (!DBL) {
        float T[N3];
        part_apply_M<TP>(Mv, xv, T);
        float2 g2[NK2 * NH];
        if constexpr (NH == N3) {
          lds_f2_at<0, NK2 * N3>(sG + t * GW, g2);
        } else {
          sfor<NK2>([&](auto KP) {
            constexpr int kp = decltype(KP)::value;
            lds_f2_at<kp * N3 + A3, NH>(sG + t * GW, g2 + kp * NH);
          });
        }
        float2 dT2[N3];
#pragma unroll
        for (int i = A3; i < B3; ++i) dT2[i] = make_float2(0.f, 0.f);
#pragma unroll
        for (int kp = 0; kp < NK2; ++kp)
#pragma unroll
          for (int i = A3; i < B3; ++i) {
            const float2 g = g2[kp * NH + (i - A3)];
            dT2[i] = __ffma2_rn(b2[kp], g, dT2[i]);
            db[kp] = __ffma2_rn(g, make_float2(T[i], T[i]), db[kp]);
          }
        float dT[N3];
#pragma unroll
        for (int i = 0; i < N3; ++i) dT[i] = (i >= A3 && i < B3) ? dT2[i].x + dT2[i].y : 0.f;
        part_outer_Q<TP>(xv, dT, Q);
      } else {
        float x1v[N1];
        if constexpr (CHU < CH) {
#pragma unroll
          for (int i = 0; i < N1; ++i) x1v[i] = sX1l[t * N1 + i];
        } else if constexpr (XB4) {
#pragma unroll
          for (int i = 0; i < N1; ++i) x1v[i] = x1g[ti * N1 + i];
        } else {
          lds_run<ti * N1, N1>(sX1l, x1v);
        }
        float2 TT[N3];  // (M x, Md x)
        float T[N3], T12[N3];
        part_apply_M2<TP>(MM, xv, x1v, TT, T12);
#pragma unroll
        for (int i = 0; i < N3; ++i) {
          T[i] = TT[i].x;
          T12[i] += TT[i].y;
        }
        float2 dG2[N3], dX2[N3];
#pragma unroll
        for (int i = A3; i < B3; ++i) dG2[i] = dX2[i] = make_float2(0.f, 0.f);
        // G (and Gt) rows in KH slices of radial pairs (bounds the live registers)
        constexpr int KH = NK2 >= 4 ? 2 : 1, KS = NK2 / KH;  // KS pairs per slice
        sfor<KH>([&](auto KHI) {
          constexpr int kh = decltype(KHI)::value;
          float2 g2[KS * NH];
          [[maybe_unused]] float2 gt2[GT ? KS * NH : 1];
          if constexpr (NH == N3) {
            lds_f2_at<kh * KS * N3, KS * N3>(sG + t * GW, g2);
            if constexpr (GT) lds_f2_at<kh * KS * N3, KS * N3>(sGt + t * GW, gt2);
          } else {
            sfor<KS>([&](auto KK) {
              constexpr int kk = decltype(KK)::value, kp = kh * KS + kk;
              lds_f2_at<kp * N3 + A3, NH>(sG + t * GW, g2 + kk * NH);
              if constexpr (GT) lds_f2_at<kp * N3 + A3, NH>(sGt + t * GW, gt2 + kk * NH);
            });
          }
#pragma unroll
          for (int kk = 0; kk < KS; ++kk) {
            const int kp = kh * KS + kk;
#pragma unroll
            for (int i = A3; i < B3; ++i) {
              const float2 g = g2[kk * NH + (i - A3)];
              dG2[i] = __ffma2_rn(b2[kp], g, dG2[i]);
              dX2[i] = __ffma2_rn(bd2[kp], g, dX2[i]);
              db[kp] = __ffma2_rn(g, make_float2(T12[i], T12[i]), db[kp]);
              hb[kp] = __ffma2_rn(g, make_float2(T[i], T[i]), hb[kp]);
              if constexpr (GT) {
                const float2 gt = gt2[kk * NH + (i - A3)];
                dX2[i] = __ffma2_rn(b2[kp], gt, dX2[i]);
                db[kp] = __ffma2_rn(gt, make_float2(T[i], T[i]), db[kp]);
              }
            }
          }
        });
        float dG[N3], dX[N3];
#pragma unroll
        for (int i = 0; i < N3; ++i) {
          dG[i] = (i >= A3 && i < B3) ? dG2[i].x + dG2[i].y : 0.f;
          dX[i] = (i >= A3 && i < B3) ? dX2[i].x + dX2[i].y : 0.f;
        }
        part_outer_Q<TP>(x1v, dG, Q);
        part_outer_Q<TP>(xv, dX, Q);
        part_outer_Q<TP>(xv, dG, Qh);
      }
    };
    if constexpr (CHU == CH) {
      sfor<CH>([&](auto TI) { chan(TI, 0); });
    } else {
#pragma unroll 1
      for (int tg = 0; tg < CH; tg += CHU) sfor<CHU>([&](auto TI) { chan(TI, tg); });
    }
    __syncwarp();
  }
  }  // receiver groups
  // this part's share of dY (second order: wY, hY) for the lane's edge
  float* acc = ws + L.Acc + lane * L.accs;
  float o[N2];
#pragma unroll
  for (int i = 0; i < N2; ++i) o[i] = 0.f;
  part_contract_Q<TP, L1, L2, L3>(Q, o);
#pragma unroll
  for (int i = 0; i < N2; ++i) acc[L2 * L2 + i] += o[i];
  if constexpr (DBL) {
#pragma unroll
    for (int i = 0; i < N2; ++i) o[i] = 0.f;
    part_contract_Q<TP, L1, L2, L3>(Qh, o);
#pragma unroll
    for (int i = 0; i < N2; ++i) acc[16 + L2 * L2 + i] += o[i];
  }
}

// one path of one batch: whole, or in two m3 parts when its per-lane state is
// large.  The instantiation with the gg_Theta operand (GT) keeps whole paths: its
// split form gave wrong d_vec on the warps of a CTA other than the first, for
// plans that mix l = 0 and l = 3 blocks, and no cause was found in the code.
template <int L1, int L2, int L3, int RM, bool DBL, bool GT, bool XB>
__device__ __forceinline__ void wna_path_parts(const DevPlan& pl, const DevPath& q, const WnaLay& L, float* ws,
                                               int rfirst, int nslots, int myslot, int nc, int nb, int myrow,
                                               const float* __restrict__ x, const float* __restrict__ x1,
                                               const float* __restrict__ G, const float* __restrict__ Gt, float2* db,
                                               float2* hb) {
  constexpr int N3 = 2 * L3 + 1;
  constexpr int split_nmz = XB || !DBL ? kWnaSplitNmz : kWnaSplitNmzL3;  // XB: kernels with l <= 2
  if constexpr (Tri<L1, L2, L3>::NMZ > split_nmz && N3 >= 3 && !(DBL && GT)) {
    constexpr int H = (N3 + 1) / 2;
    wna_path<L1, L2, L3, RM, DBL, GT, XB, 0, H>(pl, q, L, ws, rfirst, nslots, myslot, nc, nb, myrow, x, x1, G, Gt, db,
                                            hb);
    wna_path<L1, L2, L3, RM, DBL, GT, XB, H, N3>(pl, q, L, ws, rfirst, nslots, myslot, nc, nb, myrow, x, x1, G, Gt, db,
                                             hb);
  } else {
    wna_path<L1, L2, L3, RM, DBL, GT, XB, 0, N3>(pl, q, L, ws, rfirst, nslots, myslot, nc, nb, myrow, x, x1, G, Gt, db,
                                             hb);
  }
}

// Persistent grid of kWnWarps-warp CTAs.  A CTA takes kWnWarps work items per
// round from *counter.  Second order: an item is a window of 32 consecutive
// edges of the chunk's receiver-sorted CSR range (one edge per lane), whichever
// receivers they belong to.  First order: an item is one batch of up to 32
// edges of a receiver: item t < nc is receiver t's first batch, item t >= nc a
// further batch (list `extra`, built with seg = 32).  The warps of a CTA step
// through the paths together (one barrier per path), so the resident warps of
// an SM share one or two path bodies in the instruction caches, and the rounds
// stay balanced whatever the degrees.
// First order writes dvec (and, when given, dY [E][n_sh], db [E][R]); second
// order writes dvec.  x1 / ggv may be null (their terms vanish); Gt is used
// exactly when GT.  The counter is reset by the caller before the launch.
template <int RM, int LF, bool DBL, bool GT>
__global__ void __launch_bounds__(32 * kWnWarps, DBL ? 2 : 3)
    k_wn_adj(const __grid_constant__ DevPlan pl, int r0, int nc, const int* __restrict__ rowptr,
             const int* __restrict__ col, const float* __restrict__ vec, const float* __restrict__ ggv,
             const float* __restrict__ x, const float* __restrict__ x1, const float* __restrict__ G,
             const float* __restrict__ Gt, float* __restrict__ dvec, float* __restrict__ dYout,
             float* __restrict__ dbout, const int* __restrict__ extra, int* __restrict__ counter) {
  extern __shared__ __align__(16) float sm[];
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const WnaLay L = wna_layout_of(RM, pl.n3max, pl.n1max, DBL, GT);
  float* ws = sm + warp * L.total;
  int& s_base = *reinterpret_cast<int*>(sm + kWnWarps * L.total);  // this round's first item
  // staged buffers read where nothing was staged (radial entries k >= R) must hold zeros
  for (int i = lane; i < L.Geo; i += 32) ws[i] = 0.f;
  const int e_lo = rowptr[r0], e_hi = rowptr[r0 + nc];
  const int total = DBL ? (e_hi - e_lo + kBatchEdges - 1) / kBatchEdges : nc + extra[nc];
  // the next round is claimed while the current one runs (hides the atomic's latency)
  int claim = threadIdx.x == 0 ? atomicAdd(counter, kWnWarps) : 0;
  for (;;) {
    __syncthreads();  // every warp has read the previous round's s_base
    if (threadIdx.x == 0) {
      s_base = claim;
      claim = atomicAdd(counter, kWnWarps);
    }
    __syncthreads();
    const int t = s_base + warp;
    if (s_base >= total) break;  // uniform over the CTA
    int eb = 0, nb = 0, rfirst = 0, nslots = 0, myslot = -1;
    if constexpr (DBL) {
      if (t < total) {
        eb = e_lo + kBatchEdges * t;
        nb = min(kBatchEdges, e_hi - eb);
      }
      // the lane's receiver (chunk-local): the last node whose segment starts at or before its edge
      int rl = 0;
      if (lane < nb) {
        int lo = 0, hi = nc;  // rowptr[r0 + lo] <= e < rowptr[r0 + hi]
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if (rowptr[r0 + mid] <= eb + lane) lo = mid;
          else hi = mid;
        }
        rl = lo;
      }
      rfirst = __shfl_sync(0xffffffffu, rl, 0);
      const int rlast = __shfl_sync(0xffffffffu, rl, nb > 0 ? nb - 1 : 0);
      nslots = nb > 0 ? rlast - rfirst + 1 : 0;
      myslot = lane < nb ? rl - rfirst : -1;
    } else if (t < total) {
      int rl = t, k = 0;
      if (t >= nc) {
        rl = extra_owner(extra, nc, t - nc);
        k = 1 + (t - nc - extra[rl]);
      }
      const int e0 = rowptr[r0 + rl], e1 = rowptr[r0 + rl + 1];
      eb = e0 + kBatchEdges * k;
      nb = max(0, min(kBatchEdges, e1 - eb));
      rfirst = rl;
      nslots = nb > 0 ? 1 : 0;
      myslot = lane < nb ? 0 : -1;
    }
    const bool valid = lane < nb;
    const int e = eb + lane;
    int myrow = 0;
    float* geo = ws + L.Geo + lane * L.geos;
    float* acc = ws + L.Acc + lane * L.accs;
    if (valid) {
      myrow = col[e];
      using D1 = Dual<float, 1>;
      D1 vx(vec[3 * e]), vy(vec[3 * e + 1]), vz(vec[3 * e + 2]);
      if (DBL && ggv) {
        vx.d[0] = ggv[3 * e];
        vy.d[0] = ggv[3 * e + 1];
        vz.d[0] = ggv[3 * e + 2];
      }
      D1 nx, ny, nz, rr;
      unit(vx, vy, vz, nx, ny, nz, rr);
      D1 Y[16], b[RM];
#pragma unroll
      for (int m = 0; m < 16; ++m) Y[m] = D1(0.f);
      switch (pl.lsh) {
        case 0: sh_all<0>(nx, ny, nz, Y); break;
        case 1: sh_all<1>(nx, ny, nz, Y); break;
        case 2: sh_all<2>(nx, ny, nz, Y); break;
        default: sh_all<3>(nx, ny, nz, Y); break;
      }
      radial_basis<RM>(pl, rr, b);
#pragma unroll
      for (int m = 0; m < 16; ++m) geo[m] = Y[m].v;
#pragma unroll
      for (int k = 0; k < RM; ++k) geo[16 + k] = b[k].v;
      if constexpr (DBL) {
#pragma unroll
        for (int m = 0; m < 16; ++m) geo[16 + RM + m] = Y[m].d[0];
#pragma unroll
        for (int k = 0; k < RM; ++k) geo[32 + RM + k] = b[k].d[0];
      }
    }
#pragma unroll
    for (int m = 0; m < (DBL ? 32 : 16); ++m) acc[m] = 0.f;
    float2 db2[RM / 2], hb2[RM / 2];  // radial pairs (2kp, 2kp+1)
#pragma unroll
    for (int kp = 0; kp < RM / 2; ++kp) db2[kp] = hb2[kp] = make_float2(0.f, 0.f);
    for (int p = 0; p < pl.P; ++p) {
      const DevPath& q = pl.path[p];
      if (nb > 0) {
        switch (triple_id(q.l1, q.l2, q.l3)) {
#define TPC_CASE(a, b, c)                                                                                 \
  case triple_id(a, b, c):                                                                                \
    if constexpr (a <= LF && c <= LF)                                                                     \
      wna_path_parts<a, b, c, RM, DBL, GT, (LF <= 2)>(pl, q, L, ws, rfirst, nslots, myslot, nc, nb, myrow, x, x1, G, Gt, \
                                           db2, hb2);                                                     \
    break;
          TPC_FOR_EACH_TRIPLE(TPC_CASE)
#undef TPC_CASE
          default: break;
        }
      }
      __syncthreads();
    }
    if (valid) {
      float v[3] = {vec[3 * e], vec[3 * e + 1], vec[3 * e + 2]};
      float o3[3], db[RM], hb[RM];
#pragma unroll
      for (int kp = 0; kp < RM / 2; ++kp) {
        db[2 * kp] = db2[kp].x;
        db[2 * kp + 1] = db2[kp].y;
        hb[2 * kp] = hb2[kp].x;
        hb[2 * kp + 1] = hb2[kp].y;
      }
      if constexpr (!DBL) {
        if (dvec) {
          edge_vec_grad<RM>(pl, v, acc, db, o3);
          dvec[3 * e] = o3[0];
          dvec[3 * e + 1] = o3[1];
          dvec[3 * e + 2] = o3[2];
        }
        if (dYout)
          for (int m = 0; m < pl.n_sh; ++m) dYout[size_t(e) * pl.n_sh + m] = acc[m];
        if (dbout) {
#pragma unroll
          for (int k = 0; k < RM; ++k)
            if (k < pl.R) dbout[size_t(e) * pl.R + k] = db[k];
        }
      } else {
        float u[3] = {0.f, 0.f, 0.f};
        if (ggv) load3(ggv, e, u);
        edge_vec_grad2<RM>(pl, v, u, acc, acc + 16, db, hb, o3);
        dvec[3 * e] = o3[0];
        dvec[3 * e + 1] = o3[1];
        dvec[3 * e + 2] = o3[2];
      }
    }
    __syncwarp();
  }
}

}  // namespace tpc
