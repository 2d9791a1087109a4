// Fused edge streams: one CTA per (node, channel tile of 32*CPL) runs every path
// of the plan, one warp per path, so each edge's geometry (spherical harmonics,
// radial basis) is evaluated once per CTA and the gathered feature rows are
// staged once per batch in shared memory (cp.async, double-buffered) and shared
// by all path warps.  Each lane carries CPL channels so that the broadcast
// reads of the coupling matrix and radial basis are amortised over CPL times
// the FFMA work.
//
// Streams ("Sobek", arXiv 2607.18074, abstract: edge-local products consumed
// directly into bounded node-side state):
//   k_fwd_fused   receiver-sorted: A[r, k, p, u, m3] = sum_e b_ek sum_m1 M_e[m1][m3] x[s_e, u, m1]
//   k_send_fused  sender-sorted:   B[s, k, p, w, m1] = sum_e b_ek sum_m3 M_e[m1][m3] g[r_e, w, m3]
#pragma once

#include "streams.cuh"

namespace tpc {

constexpr int kFusedMaxWarps = 14;

__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async16_ca(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// shared-memory layout of a fused stream CTA (float offsets)
struct FzLay {
  int Y, B, S, T, X, M;
  int xw;  // staged row floats per edge
};
__device__ __forceinline__ FzLay fz_layout(int RM, int xw) {
  FzLay L;
  L.Y = 0;
  L.B = L.Y + 2 * kEdgeBatch * 16;
  L.S = L.B + 2 * kEdgeBatch * RM;
  L.T = L.S + 2 * kEdgeBatch;
  L.X = (L.T + 2 * kMaxBlocks + 3) & ~3;
  L.xw = xw;
  L.M = L.X + 2 * kEdgeBatch * L.xw;
  return L;
}

// Per-CTA tile of the gathered rows: block i gets channels [c0, c0 + width_i)
// at staged offset toff_i; written once by thread 0.
__device__ __forceinline__ void fz_tile(int nblk, const int* mul, const int* lval, int c0, int cw, int* sT) {
  if (threadIdx.x == 0) {
    int o = 0;
    for (int i = 0; i < nblk; ++i) {
      int w = min(cw, mul[i] - c0);
      if (w < 0) w = 0;
      sT[i] = o;
      sT[kMaxBlocks + i] = w;
      o += w * (2 * lval[i] + 1);
    }
  }
}

// Stage one batch: geometry (lane = edge, warp 0), the neighbour index, and the
// gathered rows src[idx[j]][block slice] (all threads, cp.async).
template <int RM>
__device__ __forceinline__ void fz_stage(const DevPlan& pl, const FzLay& L, float* sm, int buf, int jb, int nb,
                                         const int* __restrict__ nbr, const int* __restrict__ eid,
                                         const float* __restrict__ vec, const float* __restrict__ src, int src_dim,
                                         int nblk, const int* blk_off, const int* lval, int c0) {
  const int* sT = reinterpret_cast<const int*>(sm + L.T);
  if (threadIdx.x < 32 && threadIdx.x < nb) {
    const int j = threadIdx.x;
    const int e = eid ? eid[jb + j] : jb + j;
    float nx, ny, nz, r;
    unit(vec[3 * e], vec[3 * e + 1], vec[3 * e + 2], nx, ny, nz, r);
    float* Y = sm + L.Y + (buf * kEdgeBatch + j) * 16;
    switch (pl.lsh) {
      case 0: sh_all<0>(nx, ny, nz, Y); break;
      case 1: sh_all<1>(nx, ny, nz, Y); break;
      case 2: sh_all<2>(nx, ny, nz, Y); break;
      default: sh_all<3>(nx, ny, nz, Y); break;
    }
    radial_basis<RM>(pl, r, sm + L.B + (buf * kEdgeBatch + j) * RM);
    reinterpret_cast<int*>(sm + L.S)[buf * kEdgeBatch + j] = nbr[jb + j];
  }
  float* X = sm + L.X + buf * kEdgeBatch * L.xw;
  // 16-byte copies when every staged segment and row pitch is 16-byte aligned
  bool vec4 = (L.xw & 3) == 0 && (src_dim & 3) == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0;
  for (int i = 0; i < nblk && vec4; ++i) {
    const int n = 2 * lval[i] + 1;
    vec4 = ((blk_off[i] + c0 * n) & 3) == 0 && (sT[i] & 3) == 0 && ((sT[kMaxBlocks + i] * n) & 3) == 0;
  }
  for (int i = 0; i < nblk; ++i) {
    const int w = sT[kMaxBlocks + i];
    if (w <= 0) continue;
    const int n = 2 * lval[i] + 1;
    const int len = w * n;
    const int so = blk_off[i] + c0 * n, dof = sT[i];
    if (vec4) {
      const int len4 = len >> 2;
      for (int j = 0; j < nb; ++j) {
        const float* row = src + size_t(nbr[jb + j]) * src_dim + so;
        for (int o = threadIdx.x; o < len4; o += blockDim.x)
          cp_async16_ca(X + j * L.xw + dof + 4 * o, row + 4 * o);
      }
    } else {
      for (int idx = threadIdx.x; idx < nb * len; idx += blockDim.x) {
        const int j = idx / len, o = idx - j * len;
        const int s = nbr[jb + j];
        cp_async4(X + j * L.xw + dof + o, src + size_t(s) * src_dim + so + o);
      }
    }
  }
  cp_async_commit();
}

// ---------------------------------------------------------------------------
// forward: one warp = one path over the whole segment of receiver r
// ---------------------------------------------------------------------------
template <int L1, int L2, int L3, int RM, int CPL>
__device__ __forceinline__ void fwd_fused_path(const DevPlan& pl, const DevPath* pa, const FzLay& L, float* sm,
                                               int r, int rl, int c0, const int* __restrict__ rowptr,
                                               const int* __restrict__ col, const float* __restrict__ vec,
                                               const float* __restrict__ x, float* __restrict__ A) {
  using TR = Tri<L1, L2, L3>;
  constexpr int N1 = TR::N1, N3 = TR::N3, NMZ = TR::NMZ, NMZP = (NMZ + 3) & ~3, EB = kEdgeBatch;
  const int lane = lane_id();
  float acc[CPL][RM][N3];
#pragma unroll
  for (int q = 0; q < CPL; ++q)
#pragma unroll
    for (int k = 0; k < RM; ++k)
#pragma unroll
      for (int i = 0; i < N3; ++i) acc[q][k][i] = 0.f;
  bool act[CPL];
  int toff = 0;
  float* sMw = nullptr;
  if (pa) {
#pragma unroll
    for (int q = 0; q < CPL; ++q) act[q] = c0 + lane + 32 * q < pa->c_in;
    toff = reinterpret_cast<const int*>(sm + L.T)[pa->i1];
    sMw = sm + L.M + pa->smf_off;
  }
  const int e0 = rowptr[r], e1 = rowptr[r + 1];
  const int nbat = (e1 - e0 + EB - 1) / EB;
  if (nbat > 0)
    fz_stage<RM>(pl, L, sm, 0, e0, min(EB, e1 - e0), col, nullptr, vec, x, pl.dim_in, pl.n_in, pl.in_off,
                 pl.in_l, c0);
  cp_async_wait_all();
  __syncthreads();
  for (int bi = 0; bi < nbat; ++bi) {
    const int buf = bi & 1;
    const int eb = e0 + bi * EB, nb = min(EB, e1 - eb);
    if (bi + 1 < nbat)
      fz_stage<RM>(pl, L, sm, buf ^ 1, eb + EB, min(EB, e1 - eb - EB), col, nullptr, vec, x, pl.dim_in, pl.n_in,
                   pl.in_off, pl.in_l, c0);
    if (pa) {
      if (lane < nb) coupling_row<L1, L2, L3>(sm + L.Y + (buf * EB + lane) * 16 + L2 * L2, sMw + lane * NMZP);
      __syncwarp();
      const float* X = sm + L.X + buf * EB * L.xw + toff;
      for (int j = 0; j < nb; ++j) {
        float Mv[NMZP];
#pragma unroll
        for (int i = 0; i < NMZP / 4; ++i) {
          const float4 t = reinterpret_cast<const float4*>(sMw + j * NMZP)[i];
          Mv[4 * i] = t.x;
          Mv[4 * i + 1] = t.y;
          Mv[4 * i + 2] = t.z;
          Mv[4 * i + 3] = t.w;
        }
        float bv[RM];
#pragma unroll
        for (int i = 0; i < RM / 4; ++i) {
          const float4 t = reinterpret_cast<const float4*>(sm + L.B + (buf * EB + j) * RM)[i];
          bv[4 * i] = t.x;
          bv[4 * i + 1] = t.y;
          bv[4 * i + 2] = t.z;
          bv[4 * i + 3] = t.w;
        }
        const float* xj = X + j * L.xw;
#pragma unroll
        for (int q = 0; q < CPL; ++q) {
          float xv[N1];
#pragma unroll
          for (int i = 0; i < N1; ++i) xv[i] = act[q] ? xj[(lane + 32 * q) * N1 + i] : 0.f;
          float T[N3];
          apply_M<L1, L2, L3>(Mv, xv, T);
#pragma unroll
          for (int k = 0; k < RM; ++k)
#pragma unroll
            for (int i = 0; i < N3; ++i) acc[q][k][i] = fmaf(bv[k], T[i], acc[q][k][i]);
        }
      }
    }
    cp_async_wait_all();
    __syncthreads();
  }
  if (!pa) return;
  const int Kb = pl.Kb[pa->i3];
  float* Ablk = A + size_t(gridDim.x) * pl.a_pref[pa->i3];
#pragma unroll
  for (int q = 0; q < CPL; ++q) {
    if (!act[q]) continue;
    const int u = c0 + lane + 32 * q;
#pragma unroll
    for (int k = 0; k < RM; ++k) {
      if (k >= pl.R) break;
#pragma unroll
      for (int i = 0; i < N3; ++i) Ablk[size_t(rl * N3 + i) * Kb + pa->koff + k * pa->c_in + u] = acc[q][k][i];
    }
  }
}

// grid: (receivers in chunk, channel tiles); block: 32 * pl.fz_warps
template <int RM, int CPL>
__global__ void __launch_bounds__(32 * kFusedMaxWarps, 1)
    k_fwd_fused(const __grid_constant__ DevPlan pl, int r0, const int* __restrict__ rowptr,
                const int* __restrict__ col, const float* __restrict__ vec, const float* __restrict__ x,
                float* __restrict__ A) {
  extern __shared__ __align__(16) float sm[];
  const FzLay L = fz_layout(RM, pl.fz_xw_f);
  const int rl = blockIdx.x, r = r0 + rl;
  const int c0 = blockIdx.y * 32 * CPL;
  fz_tile(pl.n_in, pl.in_mul, pl.in_l, c0, 32 * CPL, reinterpret_cast<int*>(sm + L.T));
  __syncthreads();
  const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int p0 = 0; p0 < pl.P; p0 += nw) {
    const int p = p0 + warp;
    const DevPath* pa = (p < pl.P && c0 < pl.path[p].c_in) ? &pl.path[p] : nullptr;
    const int tid = pa ? triple_id(pa->l1, pa->l2, pa->l3) : -1;
    switch (tid) {
#define TPC_CASE(a, b, c)                                                                        \
  case triple_id(a, b, c):                                                                       \
    fwd_fused_path<a, b, c, RM, CPL>(pl, pa, L, sm, r, rl, c0, rowptr, col, vec, x, A);          \
    break;
      TPC_FOR_EACH_TRIPLE(TPC_CASE)
#undef TPC_CASE
      default: fwd_fused_path<0, 0, 0, RM, CPL>(pl, nullptr, L, sm, r, rl, c0, rowptr, col, vec, x, A); break;
    }
  }
}

// ---------------------------------------------------------------------------
// backward sender stream: one warp = one path over the out-edges of sender s
// ---------------------------------------------------------------------------
template <int L1, int L2, int L3, int RM, int CPL>
__device__ __forceinline__ void send_fused_path(const DevPlan& pl, const DevPath* pa, const FzLay& L, float* sm,
                                                int s, int sl, int c0, const int* __restrict__ s_rowptr,
                                                const int* __restrict__ perm, const int* __restrict__ s_recv,
                                                const float* __restrict__ vec, const float* __restrict__ g,
                                                float* __restrict__ B) {
  using TR = Tri<L1, L2, L3>;
  constexpr int N1 = TR::N1, N3 = TR::N3, NMZ = TR::NMZ, NMZP = (NMZ + 3) & ~3, EB = kEdgeBatch;
  const int lane = lane_id();
  float acc[CPL][RM][N1];
#pragma unroll
  for (int q = 0; q < CPL; ++q)
#pragma unroll
    for (int k = 0; k < RM; ++k)
#pragma unroll
      for (int i = 0; i < N1; ++i) acc[q][k][i] = 0.f;
  bool act[CPL];
  int toff = 0;
  float* sMw = nullptr;
  if (pa) {
#pragma unroll
    for (int q = 0; q < CPL; ++q) act[q] = c0 + lane + 32 * q < pa->c_out;
    toff = reinterpret_cast<const int*>(sm + L.T)[pa->i3];
    sMw = sm + L.M + pa->smf_off;
  }
  const int j0 = s_rowptr[s], j1 = s_rowptr[s + 1];
  const int nbat = (j1 - j0 + EB - 1) / EB;
  if (nbat > 0)
    fz_stage<RM>(pl, L, sm, 0, j0, min(EB, j1 - j0), s_recv, perm, vec, g, pl.dim_out, pl.n_out, pl.out_off,
                 pl.out_l, c0);
  cp_async_wait_all();
  __syncthreads();
  for (int bi = 0; bi < nbat; ++bi) {
    const int buf = bi & 1;
    const int jb = j0 + bi * EB, nb = min(EB, j1 - jb);
    if (bi + 1 < nbat)
      fz_stage<RM>(pl, L, sm, buf ^ 1, jb + EB, min(EB, j1 - jb - EB), s_recv, perm, vec, g, pl.dim_out,
                   pl.n_out, pl.out_off, pl.out_l, c0);
    if (pa) {
      if (lane < nb) coupling_row<L1, L2, L3>(sm + L.Y + (buf * EB + lane) * 16 + L2 * L2, sMw + lane * NMZP);
      __syncwarp();
      const float* G = sm + L.X + buf * EB * L.xw + toff;
      for (int j = 0; j < nb; ++j) {
        float Mv[NMZP];
#pragma unroll
        for (int i = 0; i < NMZP / 4; ++i) {
          const float4 t = reinterpret_cast<const float4*>(sMw + j * NMZP)[i];
          Mv[4 * i] = t.x;
          Mv[4 * i + 1] = t.y;
          Mv[4 * i + 2] = t.z;
          Mv[4 * i + 3] = t.w;
        }
        float bv[RM];
#pragma unroll
        for (int i = 0; i < RM / 4; ++i) {
          const float4 t = reinterpret_cast<const float4*>(sm + L.B + (buf * EB + j) * RM)[i];
          bv[4 * i] = t.x;
          bv[4 * i + 1] = t.y;
          bv[4 * i + 2] = t.z;
          bv[4 * i + 3] = t.w;
        }
        const float* gj = G + j * L.xw;
#pragma unroll
        for (int q = 0; q < CPL; ++q) {
          float gv[N3];
#pragma unroll
          for (int i = 0; i < N3; ++i) gv[i] = act[q] ? gj[(lane + 32 * q) * N3 + i] : 0.f;
          float U[N1];
          apply_Mt<L1, L2, L3>(Mv, gv, U);
#pragma unroll
          for (int k = 0; k < RM; ++k)
#pragma unroll
            for (int i = 0; i < N1; ++i) acc[q][k][i] = fmaf(bv[k], U[i], acc[q][k][i]);
        }
      }
    }
    cp_async_wait_all();
    __syncthreads();
  }
  if (!pa) return;
  const int Kx = pl.Kx[pa->i1];
  float* Bblk = B + size_t(gridDim.x) * pl.b_pref[pa->i1];
#pragma unroll
  for (int q = 0; q < CPL; ++q) {
    if (!act[q]) continue;
    const int w = c0 + lane + 32 * q;
#pragma unroll
    for (int k = 0; k < RM; ++k) {
      if (k >= pl.R) break;
#pragma unroll
      for (int i = 0; i < N1; ++i) Bblk[size_t(sl * N1 + i) * Kx + pa->kxoff + k * pa->c_out + w] = acc[q][k][i];
    }
  }
}

template <int RM, int CPL>
__global__ void __launch_bounds__(32 * kFusedMaxWarps, 1)
    k_send_fused(const __grid_constant__ DevPlan pl, int s0, const int* __restrict__ s_rowptr,
                 const int* __restrict__ perm, const int* __restrict__ s_recv, const float* __restrict__ vec,
                 const float* __restrict__ g, float* __restrict__ B) {
  extern __shared__ __align__(16) float sm[];
  const FzLay L = fz_layout(RM, pl.fz_xw_s);
  const int sl = blockIdx.x, s = s0 + sl;
  const int c0 = blockIdx.y * 32 * CPL;
  fz_tile(pl.n_out, pl.out_mul, pl.out_l, c0, 32 * CPL, reinterpret_cast<int*>(sm + L.T));
  __syncthreads();
  const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int p0 = 0; p0 < pl.P; p0 += nw) {
    const int p = p0 + warp;
    const DevPath* pa = (p < pl.P && c0 < pl.path[p].c_out) ? &pl.path[p] : nullptr;
    const int tid = pa ? triple_id(pa->l1, pa->l2, pa->l3) : -1;
    switch (tid) {
#define TPC_CASE(a, b, c)                                                                                   \
  case triple_id(a, b, c):                                                                                  \
    send_fused_path<a, b, c, RM, CPL>(pl, pa, L, sm, s, sl, c0, s_rowptr, perm, s_recv, vec, g, B);         \
    break;
      TPC_FOR_EACH_TRIPLE(TPC_CASE)
#undef TPC_CASE
      default:
        send_fused_path<0, 0, 0, RM, CPL>(pl, nullptr, L, sm, s, sl, c0, s_rowptr, perm, s_recv, vec, g, B);
        break;
    }
  }
}

}  // namespace tpc
