// Host planner: irreps parsing, selection-rule path table, real CG generation,
// workspace sizing.  Touches no device.
//
// Paths and their order follow the selection rules of "The Price of Freedom"
// (Approach: interactability of the Clebsch-Gordan tensor product); the node-side
// state sizes follow the receiver-side state of "Sobek" (arXiv 2607.18074,
// abstract).
#include <algorithm>
#include <cmath>
#include <complex>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "plan.h"
#include "wn_layout.h"
#include "workspace.h"
#include "dtheta_tc.h"

using namespace tpc;

// ---------------------------------------------------------------------------
// Real Clebsch-Gordan coefficients.
// Complex CG <l1 a l2 b | l3 c> from the Racah closed form (Condon-Shortley
// phase), mapped to the real basis with the unitary U (Y_real = U Y_complex):
//   m > 0 : Y_m = (Y^{-m} + (-1)^m Y^{m}) / sqrt2
//   m = 0 : Y_0 = Y^0
//   m < 0 : Y_m = i (Y^{m} - (-1)^m Y^{-m}) / sqrt2
//   C[m1,m2,m3] = sum_{a,b} conj(U1[m1,a]) conj(U2[m2,b]) U3[m3,a+b] <l1 a l2 b|l3 a+b>.
// The result is real or purely imaginary up to a global phase; the non-vanishing
// part is kept, normalised to sum_{m1 m2} C^2 = 1 per m3, and signed so that the
// first entry (lexicographic m1, m2, m3) above 1e-9 in magnitude is positive.
// ---------------------------------------------------------------------------
namespace {

double fact(int n) {
  double f = 1.0;
  for (int i = 2; i <= n; ++i) f *= i;
  return f;
}

double racah_cg(int j1, int m1, int j2, int m2, int J, int M) {
  if (m1 + m2 != M) return 0.0;
  if (std::abs(m1) > j1 || std::abs(m2) > j2 || std::abs(M) > J) return 0.0;
  if (!tri_ok(j1, j2, J)) return 0.0;
  double pre = std::sqrt((2.0 * J + 1.0) * fact(J + j1 - j2) * fact(J - j1 + j2) * fact(j1 + j2 - J) /
                         fact(j1 + j2 + J + 1));
  pre *= std::sqrt(fact(J + M) * fact(J - M) * fact(j1 - m1) * fact(j1 + m1) * fact(j2 - m2) *
                   fact(j2 + m2));
  double s = 0.0;
  for (int k = 0; k <= j1 + j2 + J; ++k) {
    int d[6] = {k, j1 + j2 - J - k, j1 - m1 - k, j2 + m2 - k, J - j2 + m1 + k, J - j1 - m2 + k};
    bool ok = true;
    for (int i = 0; i < 6; ++i) ok = ok && d[i] >= 0;
    if (!ok) continue;
    double den = 1.0;
    for (int i = 0; i < 6; ++i) den *= fact(d[i]);
    s += ((k & 1) ? -1.0 : 1.0) / den;
  }
  return pre * s;
}

using cplx = std::complex<double>;

void real_basis_U(int l, std::vector<cplx>& U) {
  int n = 2 * l + 1;
  U.assign(n * n, cplx(0, 0));
  const double r2 = 1.0 / std::sqrt(2.0);
  for (int m = -l; m <= l; ++m) {
    int row = m + l;
    double sgn = (std::abs(m) & 1) ? -1.0 : 1.0;
    if (m > 0) {
      U[row * n + (-m + l)] = cplx(r2, 0);
      U[row * n + (m + l)] = cplx(sgn * r2, 0);
    } else if (m == 0) {
      U[row * n + l] = cplx(1, 0);
    } else {
      U[row * n + (m + l)] = cplx(0, r2);
      U[row * n + (-m + l)] = cplx(0, -sgn * r2);
    }
  }
}

// returns 0 on success
int real_cg_triple(int l1, int l2, int l3, double* out) {
  const int n1 = 2 * l1 + 1, n2 = 2 * l2 + 1, n3 = 2 * l3 + 1;
  std::vector<cplx> U1, U2, U3;
  real_basis_U(l1, U1);
  real_basis_U(l2, U2);
  real_basis_U(l3, U3);
  std::vector<cplx> C(n1 * n2 * n3, cplx(0, 0));
  for (int i1 = 0; i1 < n1; ++i1)
    for (int i2 = 0; i2 < n2; ++i2)
      for (int i3 = 0; i3 < n3; ++i3) {
        cplx s(0, 0);
        for (int a = -l1; a <= l1; ++a)
          for (int b = -l2; b <= l2; ++b) {
            int c = a + b;
            if (c < -l3 || c > l3) continue;
            double cg = racah_cg(l1, a, l2, b, l3, c);
            if (cg == 0.0) continue;
            s += std::conj(U1[i1 * n1 + a + l1]) * std::conj(U2[i2 * n2 + b + l2]) *
                 U3[i3 * n3 + c + l3] * cg;
          }
        C[(i1 * n2 + i2) * n3 + i3] = s;
      }
  double nre = 0, nim = 0;
  for (auto& c : C) {
    nre += c.real() * c.real();
    nim += c.imag() * c.imag();
  }
  const bool use_re = nre >= nim;
  double nrm = 0;
  for (size_t i = 0; i < C.size(); ++i) {
    out[i] = use_re ? C[i].real() : C[i].imag();
    nrm += out[i] * out[i];
  }
  if (nrm <= 0) return 1;
  double scale = std::sqrt(double(n3) / nrm);
  int first = -1;
  for (size_t i = 0; i < C.size(); ++i) {
    out[i] *= scale;
    if (first < 0 && std::fabs(out[i]) > 1e-9) first = int(i);
  }
  if (first < 0) return 1;
  if (out[first] < 0)
    for (size_t i = 0; i < C.size(); ++i) out[i] = -out[i];
  for (size_t i = 0; i < C.size(); ++i)
    if (std::fabs(out[i]) < 1e-13) out[i] = 0.0;
  // self-check: orthonormal columns (per m3) and the structural zero pattern
  for (int a = 0; a < n3; ++a)
    for (int b = 0; b < n3; ++b) {
      double s = 0;
      for (int i = 0; i < n1 * n2; ++i) s += out[i * n3 + a] * out[i * n3 + b];
      if (std::fabs(s - (a == b ? 1.0 : 0.0)) > 1e-12) return 2;
    }
  for (int i1 = 0; i1 < n1; ++i1)
    for (int i2 = 0; i2 < n2; ++i2)
      for (int i3 = 0; i3 < n3; ++i3)
        if (out[(i1 * n2 + i2) * n3 + i3] != 0.0 && !cg_struct_nz(l1, l2, l3, i1, i2, i3)) return 3;
  return 0;
}

std::once_flag g_cg_once;
int g_cg_status = 0;
float g_cg_f32[kCgTotal];

}  // namespace

int tpc::generate_cg_table(double* dense) {
  for (int a = 0; a <= kMaxL; ++a)
    for (int b = 0; b <= kMaxL; ++b)
      for (int c = 0; c <= kMaxL; ++c) {
        if (!tri_ok(a, b, c)) continue;
        int st = real_cg_triple(a, b, c, dense + cg_offset(a, b, c));
        if (st) return st;
      }
  return 0;
}

const float* tpc::cg_table_f32() {
  std::call_once(g_cg_once, [] {
    std::vector<double> d(kCgTotal);
    g_cg_status = generate_cg_table(d.data());
    for (int i = 0; i < kCgTotal; ++i) g_cg_f32[i] = float(d[i]);
  });
  return g_cg_status == 0 ? g_cg_f32 : nullptr;
}

// ---------------------------------------------------------------------------
// irreps parsing
// ---------------------------------------------------------------------------
namespace {
struct Blk {
  int mul, l, p;
};

int parse_irreps(const char* s, std::vector<Blk>& out) {
  out.clear();
  if (!s) return TPCONV_ERR_INVALID_ARG;
  std::string str;
  for (const char* c = s; *c; ++c)
    if (*c != ' ') str.push_back(*c);
  if (str.empty()) return TPCONV_ERR_BAD_IRREPS;
  size_t pos = 0;
  while (pos <= str.size()) {
    size_t end = str.find('+', pos);
    if (end == std::string::npos) end = str.size();
    std::string tok = str.substr(pos, end - pos);
    size_t x = tok.find('x');
    if (x == std::string::npos || x == 0 || x + 2 > tok.size()) return TPCONV_ERR_BAD_IRREPS;
    std::string smul = tok.substr(0, x), sl = tok.substr(x + 1, tok.size() - x - 2);
    char par = tok.back();
    if (sl.empty() || (par != 'e' && par != 'o')) return TPCONV_ERR_BAD_IRREPS;
    for (char c : smul)
      if (c < '0' || c > '9') return TPCONV_ERR_BAD_IRREPS;
    for (char c : sl)
      if (c < '0' || c > '9') return TPCONV_ERR_BAD_IRREPS;
    if (smul.size() > 6 || sl.size() > 3) return TPCONV_ERR_UNSUPPORTED;
    Blk b{std::atoi(smul.c_str()), std::atoi(sl.c_str()), par == 'e' ? 1 : -1};
    if (b.mul < 1) return TPCONV_ERR_BAD_IRREPS;
    if (b.l > kMaxL) return TPCONV_ERR_UNSUPPORTED;
    out.push_back(b);
    if (end == str.size()) break;
    pos = end + 1;
  }
  if (out.size() > size_t(kMaxBlocks)) return TPCONV_ERR_UNSUPPORTED;
  return TPCONV_OK;
}
}  // namespace

// ---------------------------------------------------------------------------
// public host API
// ---------------------------------------------------------------------------
extern "C" {

void tpconv_default_options(tpconv_options* opt) {
  if (!opt) return;
  std::memset(opt, 0, sizeof(*opt));
  opt->radial = TPCONV_RADIAL_BESSEL_COS;
  opt->radial_p0 = 5.0;
  opt->radial_p1 = 0.0;
  opt->gemm = TPCONV_GEMM_FP32;
  opt->workspace_cap = 0;
  opt->validate = 0;
  opt->family = TPCONV_FAMILY_FULL;
}

const char* tpconv_status_string(int st) {
  switch (st) {
    case TPCONV_OK: return "ok";
    case TPCONV_ERR_INVALID_ARG: return "invalid argument";
    case TPCONV_ERR_BAD_IRREPS: return "irreps string does not parse";
    case TPCONV_ERR_UNSUPPORTED: return "unsupported size or degree";
    case TPCONV_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case TPCONV_ERR_CUDA: return "CUDA runtime error";
    case TPCONV_ERR_GRAPH_INVALID: return "graph invalid";
    case TPCONV_ERR_TIMEOUT: return "device wait timed out";
    case TPCONV_ERR_INTERNAL: return "internal self-check failed";
    default: return "unknown status";
  }
}

int tpconv_plan_create(tpconv_plan** out, const char* irreps_in, int l_sh_max,
                       const char* irreps_out, int R, const tpconv_options* opt) {
  if (!out) return TPCONV_ERR_INVALID_ARG;
  *out = nullptr;
  if (!irreps_in || !irreps_out) return TPCONV_ERR_INVALID_ARG;
  if (l_sh_max < 0 || R < 1) return TPCONV_ERR_INVALID_ARG;
  if (l_sh_max > kMaxL || R > kMaxR) return TPCONV_ERR_UNSUPPORTED;
  tpconv_options o;
  tpconv_default_options(&o);
  if (opt) o = *opt;
  if (o.radial != TPCONV_RADIAL_GAUSSIAN && o.radial != TPCONV_RADIAL_BESSEL_COS)
    return TPCONV_ERR_INVALID_ARG;
  if (o.gemm < TPCONV_GEMM_FP32 || o.gemm > TPCONV_GEMM_SIMT) return TPCONV_ERR_INVALID_ARG;
  if (o.gemm == 2) return TPCONV_ERR_UNSUPPORTED;  // no half-precision operand mode (see tpconv.h)
  if (o.family != TPCONV_FAMILY_FULL && o.family != TPCONV_FAMILY_CHANNELWISE) return TPCONV_ERR_INVALID_ARG;
  if (o.radial == TPCONV_RADIAL_BESSEL_COS && !(o.radial_p0 > 0)) return TPCONV_ERR_INVALID_ARG;
  if (o.radial == TPCONV_RADIAL_GAUSSIAN && !(o.radial_p1 > o.radial_p0)) return TPCONV_ERR_INVALID_ARG;

  std::vector<Blk> bin, bout;
  int st = parse_irreps(irreps_in, bin);
  if (st) return st;
  st = parse_irreps(irreps_out, bout);
  if (st) return st;
  if (!cg_table_f32()) return TPCONV_ERR_INTERNAL;

  tpconv_plan* p = new (std::nothrow) tpconv_plan();
  if (!p) return TPCONV_ERR_INTERNAL;
  DevPlan& d = p->dp;
  std::memset(&d, 0, sizeof(d));
  d.R = R;
  d.lsh = l_sh_max;
  d.n_sh = (l_sh_max + 1) * (l_sh_max + 1);
  d.radial = o.radial;
  d.rp0 = float(o.radial_p0);
  d.rp1 = float(o.radial_p1);
  if (o.radial == TPCONV_RADIAL_GAUSSIAN) {
    double D = R > 1 ? (o.radial_p1 - o.radial_p0) / (R - 1) : (o.radial_p1 - o.radial_p0);
    d.rc0 = float(D);
    d.rc1 = float(1.0 / D);
  } else {
    d.rc0 = float(3.14159265358979323846 / o.radial_p0);
    d.rc1 = float(std::sqrt(2.0 / o.radial_p0));
  }
  d.n_in = int(bin.size());
  d.n_out = int(bout.size());
  int off = 0;
  for (int i = 0; i < d.n_in; ++i) {
    d.in_l[i] = bin[i].l;
    d.in_mul[i] = bin[i].mul;
    d.in_off[i] = off;
    off += bin[i].mul * (2 * bin[i].l + 1);
    d.max_c_in = std::max(d.max_c_in, bin[i].mul);
  }
  d.dim_in = off;
  off = 0;
  for (int i = 0; i < d.n_out; ++i) {
    d.out_l[i] = bout[i].l;
    d.out_mul[i] = bout[i].mul;
    d.out_off[i] = off;
    off += bout[i].mul * (2 * bout[i].l + 1);
    d.max_c_out = std::max(d.max_c_out, bout[i].mul);
  }
  d.dim_out = off;

  int P = 0;
  int64_t toff = 0;
  for (int i3 = 0; i3 < d.n_out; ++i3)
    for (int i1 = 0; i1 < d.n_in; ++i1)
      for (int l2 = 0; l2 <= l_sh_max; ++l2) {
        const Blk &b1 = bin[i1], &b3 = bout[i3];
        if (!tri_ok(b1.l, l2, b3.l)) continue;
        if (b1.p * ((l2 & 1) ? -1 : 1) != b3.p) continue;
        if (P >= kMaxPaths) {
          delete p;
          return TPCONV_ERR_UNSUPPORTED;
        }
        if (o.family == TPCONV_FAMILY_CHANNELWISE && b1.mul != b3.mul) {  // one weight per channel
          delete p;
          return TPCONV_ERR_INVALID_ARG;
        }
        DevPath& q = d.path[P++];
        q.l1 = int8_t(b1.l);
        q.l2 = int8_t(l2);
        q.l3 = int8_t(b3.l);
        q.i1 = int16_t(i1);
        q.i3 = int16_t(i3);
        q.c_in = b1.mul;
        q.c_out = b3.mul;
        q.in_off = d.in_off[i1];
        q.out_off = d.out_off[i3];
        q.theta_off = toff;
        q.koff = d.Kb[i3];
        d.Kb[i3] += R * b1.mul;
        q.kxoff = d.Kx[i1];
        d.Kx[i1] += R * b3.mul;
        toff += int64_t(R) * b1.mul * (o.family == TPCONV_FAMILY_CHANNELWISE ? 1 : b3.mul);
      }
  d.P = P;
  d.family = o.family;
  d.rm = R <= 8 ? 8 : 16;  // radial registers per lane; entries k >= R stay zero
  int sm = 0, sm2 = 0;
  for (int i = 0; i < P; ++i) {
    DevPath& q = d.path[i];
    q.nmz = m_count(q.l1, q.l2, q.l3);
    q.sm_off = sm;
    sm += kEdgeBatch * (q.nmz + 2 * d.rm + 1 + (2 * q.l2 + 1));
    q.sm_off2 = sm2;
    sm2 += kEdgeBatch * (2 * q.nmz + 4 * d.rm + 1 + 2 * (2 * q.l2 + 1));
  }
  d.sm_floats = sm;
  d.sm_floats2 = sm2;
  // warp-per-node streams
  {
    bool ok = true;  // 16-byte staging of rows and channel groups of four (adjoint streams)
    for (int i = 0; i < d.n_in; ++i) ok = ok && (d.in_mul[i] % 4 == 0);
    for (int i = 0; i < d.n_out; ++i) ok = ok && (d.Kb[i] % 4 == 0);
    d.wn_ok = ok;
    d.n3max = 1;
    d.n1max = 1;
    d.nmz_max = 1;
    for (int i = 0; i < P; ++i) {
      d.n3max = std::max(d.n3max, 2 * int(d.path[i].l3) + 1);
      d.n1max = std::max(d.n1max, 2 * int(d.path[i].l1) + 1);
      d.nmz_max = std::max(d.nmz_max, int(d.path[i].nmz));
    }
  }
  // warp-per-node streams: kernels instantiated for feature degrees <= 2 (radial
  // width 8) or <= 3; two channels per lane when every path has >= 64 channels
  {
    int lmax = 0, cmin = 1 << 30;
    for (int i = 0; i < P; ++i) {
      lmax = std::max(lmax, std::max(int(d.path[i].l1), int(d.path[i].l3)));
      cmin = std::min(cmin, std::min(d.path[i].c_in, d.path[i].c_out));
    }
    d.wn_lf = (d.rm == 8 && lmax <= 2) ? 2 : 3;
    d.wn_cpl = (d.wn_lf == 2 && cmin >= 64) ? 2 : 1;
    d.wn_smem_f = wn_smem_bytes(d.rm, d.wn_cpl, d.n1max, d.nmz_max, false, false);
    d.wn_smem_s = wn_smem_bytes(d.rm, d.wn_cpl, d.n3max, d.nmz_max, false, false);
    d.wn_smem_f2 = wn_smem_bytes(d.rm, 1, d.n1max, d.nmz_max, true, true);
    d.wn_smem_s2 = wn_smem_bytes(d.rm, 1, d.n3max, d.nmz_max, true, false);
    d.wn_smem_adj = wna_smem_bytes(d.rm, d.n3max, d.n1max, false, false);
    d.wn_smem_dadj = wna_smem_bytes(d.rm, d.n3max, d.n1max, true, false);
    const int dadj_gt = wna_smem_bytes(d.rm, d.n3max, d.n1max, true, true);  // launcher computes it again
    const int mx = std::max(std::max(std::max(d.wn_smem_f, d.wn_smem_s), std::max(d.wn_smem_f2, d.wn_smem_s2)),
                            std::max(std::max(d.wn_smem_adj, d.wn_smem_dadj), dadj_gt));
    if (mx > 227 * 1024) {
      delete p;
      return TPCONV_ERR_UNSUPPORTED;
    }
  }
  // the per-path adjoint streams serve the plans whose rows cannot be staged 16 bytes at a time
  if (!d.wn_ok && size_t(std::max(sm, sm2)) * 4 > 227 * 1024) {
    delete p;
    return TPCONV_ERR_UNSUPPORTED;
  }
  d.a_pref[0] = 0;
  for (int i3 = 0; i3 < d.n_out; ++i3) d.a_pref[i3 + 1] = d.a_pref[i3] + int64_t(2 * d.out_l[i3] + 1) * d.Kb[i3];
  d.b_pref[0] = 0;
  for (int i1 = 0; i1 < d.n_in; ++i1) d.b_pref[i1 + 1] = d.b_pref[i1] + int64_t(2 * d.in_l[i1] + 1) * d.Kx[i1];
  p->opt = o;
  p->theta_numel = size_t(toff);
  p->a_floats = d.a_pref[d.n_out];
  p->b_floats = d.b_pref[d.n_in];
  *out = p;
  return TPCONV_OK;
}

int tpconv_plan_destroy(tpconv_plan* plan) {
  delete plan;
  return TPCONV_OK;
}

int tpconv_plan_info(const tpconv_plan* plan, int* n_paths, int* dim_in, int* dim_out, int* n_sh,
                     size_t* theta_numel) {
  if (!plan) return TPCONV_ERR_INVALID_ARG;
  if (n_paths) *n_paths = plan->dp.P;
  if (dim_in) *dim_in = plan->dp.dim_in;
  if (dim_out) *dim_out = plan->dp.dim_out;
  if (n_sh) *n_sh = plan->dp.n_sh;
  if (theta_numel) *theta_numel = plan->theta_numel;
  return TPCONV_OK;
}

int tpconv_plan_path(const tpconv_plan* plan, int i, int* l1, int* l2, int* l3, int* c_in,
                     int* c_out, size_t* theta_offset) {
  if (!plan || i < 0 || i >= plan->dp.P) return TPCONV_ERR_INVALID_ARG;
  const DevPath& q = plan->dp.path[i];
  if (l1) *l1 = q.l1;
  if (l2) *l2 = q.l2;
  if (l3) *l3 = q.l3;
  if (c_in) *c_in = q.c_in;
  if (c_out) *c_out = q.c_out;
  if (theta_offset) *theta_offset = size_t(q.theta_off);
  return TPCONV_OK;
}

int tpconv_cg_coefficients(int l1, int l2, int l3, double* out) {
  if (!out) return TPCONV_ERR_INVALID_ARG;
  if (l1 < 0 || l2 < 0 || l3 < 0 || l1 > kMaxL || l2 > kMaxL || l3 > kMaxL || !tri_ok(l1, l2, l3))
    return TPCONV_ERR_UNSUPPORTED;
  return real_cg_triple(l1, l2, l3, out) == 0 ? TPCONV_OK : TPCONV_ERR_INTERNAL;
}

int tpconv_workspace_size(const tpconv_plan* plan, int op, int64_t N, int64_t E, size_t* bytes) {
  if (!plan || !bytes || N < 0 || E < 0) return TPCONV_ERR_INVALID_ARG;
  WsLayout L;
  int st = ws_layout(*plan, op, N, E, &L);
  if (st) return st;
  *bytes = L.total;
  return TPCONV_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// workspace layout
// ---------------------------------------------------------------------------
static size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

int tpc::ws_layout(const tpconv_plan& p, int op, int64_t N, int64_t E, WsLayout* L) {
  std::memset(L, 0, sizeof(*L));
  if (E >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return TPCONV_ERR_UNSUPPORTED;
  size_t off = 0;
  if (op == TPCONV_OP_TRANSPOSE) {
    L->off_cursor = off;
    off = align256(off + size_t(N + 1) * 4);
    L->off_scan = off;
    off = align256(off + size_t((N + 1 + 1023) / 1024 + 2) * 4);
    L->off_tmp = off;
    off = align256(off + size_t(E) * 4);
    L->total = off;
    return TPCONV_OK;
  }
  int64_t per_node;  // floats of node-side state per node
  int64_t state_max = std::max(p.a_floats, p.b_floats);
  if (op == TPCONV_OP_FORWARD) per_node = p.a_floats;
  else if (op == TPCONV_OP_BACKWARD) per_node = state_max;
  else if (op == TPCONV_OP_DOUBLE_BACKWARD) per_node = 2 * state_max;
  else return TPCONV_ERR_INVALID_ARG;
  int64_t Nc = N;
  if (p.opt.workspace_cap > 0 && per_node > 0) {
    int64_t fit = int64_t(p.opt.workspace_cap / (size_t(per_node) * 4));
    if (fit < 1) fit = 1;
    if (fit < Nc) Nc = fit;
  }
  if (Nc < 1) Nc = 1;
  L->chunk_nodes = Nc;
  L->off_state = off;
  L->state_bytes = size_t(Nc) * size_t(per_node) * 4;
  off = align256(off + L->state_bytes);
  L->off_theta = off;
  const bool tc = p.dp.family == TPCONV_FAMILY_FULL && (p.opt.gemm == TPCONV_GEMM_FP32 || p.opt.gemm == TPCONV_GEMM_TF32);
  const int nreg = theta_region_count(op, tc, p.opt.gemm == TPCONV_GEMM_FP32);
  L->theta_bytes = align256(((p.theta_numel + 63) & ~size_t(63)) * 4 * size_t(nreg));
  off = align256(off + L->theta_bytes);
  L->off_pack = off;
  L->pack_bytes = align256(size_t(Nc) * size_t(p.dp.dim_out) * 4);
  off = align256(off + L->pack_bytes);
  L->off_lists = off;
  L->list_ints = work_list_ints(Nc);
  off = align256(off + size_t(kWorkLists) * L->list_ints * 4);
  if (tc && op != TPCONV_OP_FORWARD && dtheta_tc_shape_ok(p.dp)) {
    L->off_xt = off;
    L->xt_bytes = align256(dtheta_tc_xt_floats(p.dp, Nc) * 4);
    off += L->xt_bytes;
    L->off_part = off;
    L->part_bytes = align256(dtheta_tc_partial_floats(p.dp) * 4);
    off += L->part_bytes;
  }
  L->total = off;
  return TPCONV_OK;
}
