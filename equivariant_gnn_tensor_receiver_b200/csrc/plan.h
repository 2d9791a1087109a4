// Internal plan structures shared by the host planner and the device kernels.
//
// The plan is the path table of the tensor-product convolution: every allowed
// (input block i1, SH degree l2, output block i3) triple under the selection
// rules of "The Price of Freedom" (Approach), with the offsets the kernels use
// to address features, Theta and the node-side state of the streaming schedule
// of "Sobek" (arXiv 2607.18074, abstract).
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/tpconv.h"

namespace tpc {

constexpr int kMaxL = 3;        // highest feature / SH degree handled by the kernels
constexpr int kMaxR = 16;       // highest radial basis size
constexpr int kMaxPaths = 48;
constexpr int kMaxBlocks = 12;

// --- compile-time layout of the dense real-CG table of all triples with l <= 3 ---
constexpr bool tri_ok(int a, int b, int c) { return a - b <= c && b - a <= c && c <= a + b; }
constexpr int cg_size(int a, int b, int c) { return (2 * a + 1) * (2 * b + 1) * (2 * c + 1); }
constexpr int cg_offset(int l1, int l2, int l3) {
  int off = 0;
  for (int a = 0; a <= kMaxL; ++a)
    for (int b = 0; b <= kMaxL; ++b)
      for (int c = 0; c <= kMaxL; ++c) {
        if (a == l1 && b == l2 && c == l3) return off;
        if (tri_ok(a, b, c)) off += cg_size(a, b, c);
      }
  return -1;
}
constexpr int cg_total() {
  int off = 0;
  for (int a = 0; a <= kMaxL; ++a)
    for (int b = 0; b <= kMaxL; ++b)
      for (int c = 0; c <= kMaxL; ++c)
        if (tri_ok(a, b, c)) off += cg_size(a, b, c);
  return off;
}
constexpr int kCgTotal = cg_total();

constexpr int iabs(int v) { return v < 0 ? -v : v; }
// Structural zero pattern of the real CG tensor (indices i = m + l).  In the
// real basis |m3| must equal |m1|+|m2| or ||m1|-|m2||, and the sine/cosine type
// of m3 is fixed by those of m1, m2 and by the parity of l1+l2+l3.  Entries for
// which this returns false are zero; the host generator verifies it.
constexpr bool cg_struct_nz(int l1, int l2, int l3, int i1, int i2, int i3) {
  int m1 = i1 - l1, m2 = i2 - l2, m3 = i3 - l3;
  int a1 = iabs(m1), a2 = iabs(m2), a3 = iabs(m3);
  if (a3 != a1 + a2 && a3 != iabs(a1 - a2)) return false;
  int t1 = m1 < 0, t2 = m2 < 0, t3 = m3 < 0;
  int want = ((l1 + l2 + l3) % 2 == 0) ? (t1 ^ t2) : !(t1 ^ t2);
  return t3 == want;
}

// Structural nonzeros of the coupling matrix M[m1][m3] = sum_m2 C[m1,m2,m3] Y[m2]
// (edge-dependent, channel-independent); kernels store only these entries.
constexpr bool m_struct_nz(int l1, int l2, int l3, int i1, int i3) {
  for (int i2 = 0; i2 < 2 * l2 + 1; ++i2)
    if (cg_struct_nz(l1, l2, l3, i1, i2, i3)) return true;
  return false;
}
constexpr int m_index(int l1, int l2, int l3, int i1, int i3) {
  int c = 0;
  for (int a = 0; a < 2 * l1 + 1; ++a)
    for (int b = 0; b < 2 * l3 + 1; ++b) {
      if (a == i1 && b == i3) return c;
      if (m_struct_nz(l1, l2, l3, a, b)) ++c;
    }
  return -1;
}
constexpr int m_count(int l1, int l2, int l3) {
  int c = 0;
  for (int a = 0; a < 2 * l1 + 1; ++a)
    for (int b = 0; b < 2 * l3 + 1; ++b)
      if (m_struct_nz(l1, l2, l3, a, b)) ++c;
  return c;
}

constexpr int kEdgeBatch = 16;  // edges staged per warp batch in the edge streams

// --- per-path and per-plan descriptors passed to kernels by value ---
struct DevPath {
  int8_t l1, l2, l3, pad;
  int16_t i1, i3;
  int32_t c_in, c_out;
  int32_t in_off, out_off;  // feature offsets of blocks i1 / i3
  int32_t koff;             // A / G column of (k=0, u=0) in output block i3: koff + k*c_in + u
  int32_t kxoff;            // B column of (k=0, w=0) in input block i1: kxoff + k*c_out + w
  int64_t theta_off;        // start of Theta[p] ([R][c_in][c_out])
  int32_t nmz;              // m_count(l1, l2, l3)
  int32_t sm_off;           // float offset of this path's warp scratch (per-path adjoint stream)
  int32_t sm_off2;          // same for the per-path double-backward adjoint stream
};

struct DevPlan {
  int P, R, lsh, n_sh, dim_in, dim_out;
  int radial;
  float rp0, rp1, rc0, rc1;  // radial parameters and derived constants
  int n_in, n_out;           // number of input / output blocks
  int in_l[kMaxBlocks], in_mul[kMaxBlocks], in_off[kMaxBlocks];
  int out_l[kMaxBlocks], out_mul[kMaxBlocks], out_off[kMaxBlocks];
  int Kb[kMaxBlocks];               // columns of the A / G block of output block i3
  int64_t a_pref[kMaxBlocks + 1];   // floats per node before block i3 (sum n3 * Kb)
  int Kx[kMaxBlocks];               // columns of the B block of input block i1
  int64_t b_pref[kMaxBlocks + 1];   // floats per node before block i1 (sum n1 * Kx)
  int max_c_in, max_c_out;
  int rm;                           // radial registers per lane (8 or 16) >= R
  int sm_floats;                    // dynamic smem floats of the per-path adjoint stream
  int sm_floats2;                   // the same for its double-backward form
  int wn_ok;                        // rows stageable 16 bytes at a time (channel counts multiple of 4)
  int n3max, n1max;                 // largest 2l3+1 / 2l1+1 over the paths
  int nmz_max;                      // largest compact coupling matrix over the paths
  int wn_lf;                        // warp-per-node streams: bound on l1, l3 of the instantiation (2 or 3)
  int wn_cpl;                       // channels per lane of their first-order channel-lane forms (1 or 2)
  int wn_smem_f, wn_smem_s;         // dynamic smem bytes: receiver / sender form, first order
  int wn_smem_f2, wn_smem_s2;       // the same, second order
  int wn_smem_adj, wn_smem_dadj;    // receiver adjoint streams, first / second order
  int family;                       // TPCONV_FAMILY_*: Theta[p] is R x C_in x C_out or R x C
  DevPath path[kMaxPaths];
};

}  // namespace tpc

struct tpconv_plan {
  tpc::DevPlan dp;
  tpconv_options opt;
  size_t theta_numel;
  int64_t a_floats;  // A / G floats per node (Afl)
  int64_t b_floats;  // B floats per node
};

namespace tpc {
// Host CG generator (fp64, Racah formula mapped to the real basis).
int generate_cg_table(double* out_dense /* kCgTotal */);
// Float copy of the table, generated once per process.
const float* cg_table_f32();
}  // namespace tpc
