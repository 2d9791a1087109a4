// Device-side building blocks shared by all kernels of the library:
//  - forward-mode dual numbers (nested for second derivatives), so that the
//    spherical harmonics and radial basis give exact Jacobians / Hessian-vector
//    products in registers without separate derivative code;
//  - real spherical harmonics Y_l (l <= 3, component normalisation, m = -l..l,
//    no Condon-Shortley sign, Y_1 = sqrt3 (y, z, x)/r);
//  - the two radial bases (Gaussian; Bessel with cosine cutoff);
//  - the dense real-CG table of every triple with l <= 3 in __constant__ memory,
//    read at compile-time offsets so that the coupling compiles to FFMA with
//    constant-bank operands, and its structural zeros are pruned at compile time.
//
// The coupling is the Clebsch-Gordan tensor product of "The Price of Freedom"
// (Approach); the radial projection and spherical-harmonic coupling are the two
// edge-local factors named in the abstract of "Sobek" (arXiv 2607.18074).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>
#include <utility>

#include "plan.h"

namespace tpc {

// One copy per translation unit (no relocatable device code); each unit that
// uses it defines an uploader with TPC_DEFINE_CG_UPLOADER.
static __constant__ float c_cg[kCgTotal];

#define TPC_DEFINE_CG_UPLOADER(name)                                         \
  cudaError_t name(const float* table) {                                     \
    return cudaMemcpyToSymbol(tpc::c_cg, table, sizeof(float) * tpc::kCgTotal); \
  }

// compile-time loops: f(std::integral_constant<int, i>) for i = 0..N-1
template <class F, int... I>
__device__ __forceinline__ void sfor_(F& f, std::integer_sequence<int, I...>) {
  (f(std::integral_constant<int, I>{}), ...);
}
template <int N, class F>
__device__ __forceinline__ void sfor(F&& f) {
  sfor_(f, std::make_integer_sequence<int, N>{});
}

// Compile-time structure of one CG triple: structural nonzeros of C and of the
// coupling matrix M[m1][m3] = sum_m2 C[m1,m2,m3] Y[m2], and the compact index of
// each nonzero M entry.
template <int L1, int L2, int L3>
struct Tri {
  static constexpr int N1 = 2 * L1 + 1, N2 = 2 * L2 + 1, N3 = 2 * L3 + 1;
  static constexpr int OFF = cg_offset(L1, L2, L3);
  struct Tab {
    bool cg[N1][N2][N3];
    bool m[N1][N3];
    int mi[N1][N3];
    int nmz;
  };
  static constexpr Tab make() {
    Tab t{};
    int c = 0;
    for (int a = 0; a < N1; ++a)
      for (int b = 0; b < N3; ++b) {
        bool any = false;
        for (int i2 = 0; i2 < N2; ++i2) {
          t.cg[a][i2][b] = cg_struct_nz(L1, L2, L3, a, i2, b);
          any = any || t.cg[a][i2][b];
        }
        t.m[a][b] = any;
        t.mi[a][b] = any ? c++ : -1;
      }
    t.nmz = c;
    return t;
  }
  static constexpr Tab tab = make();
  static constexpr int NMZ = tab.nmz;
  template <int I1, int I2, int I3>
  static __device__ __forceinline__ float cg() {
    return c_cg[OFF + (I1 * N2 + I2) * N3 + I3];
  }
};

// ---------------------------------------------------------------------------
// dual numbers: value plus N directional derivatives (S may itself be a Dual)
// ---------------------------------------------------------------------------
template <class S, int N>
struct Dual {
  S v;
  S d[N];
  __device__ __forceinline__ Dual() {}
  __device__ __forceinline__ Dual(float s) : v(s) {
#pragma unroll
    for (int i = 0; i < N; ++i) d[i] = S(0.f);
  }
};

__device__ __forceinline__ float val(float a) { return a; }
template <class S, int N>
__device__ __forceinline__ float val(const Dual<S, N>& a) { return val(a.v); }

template <class S, int N>
__device__ __forceinline__ Dual<S, N> operator+(const Dual<S, N>& a, const Dual<S, N>& b) {
  Dual<S, N> r;
  r.v = a.v + b.v;
#pragma unroll
  for (int i = 0; i < N; ++i) r.d[i] = a.d[i] + b.d[i];
  return r;
}
template <class S, int N>
__device__ __forceinline__ Dual<S, N> operator-(const Dual<S, N>& a, const Dual<S, N>& b) {
  Dual<S, N> r;
  r.v = a.v - b.v;
#pragma unroll
  for (int i = 0; i < N; ++i) r.d[i] = a.d[i] - b.d[i];
  return r;
}
template <class S, int N>
__device__ __forceinline__ Dual<S, N> operator-(const Dual<S, N>& a) {
  Dual<S, N> r;
  r.v = -a.v;
#pragma unroll
  for (int i = 0; i < N; ++i) r.d[i] = -a.d[i];
  return r;
}
template <class S, int N>
__device__ __forceinline__ Dual<S, N> operator*(const Dual<S, N>& a, const Dual<S, N>& b) {
  Dual<S, N> r;
  r.v = a.v * b.v;
#pragma unroll
  for (int i = 0; i < N; ++i) r.d[i] = a.v * b.d[i] + a.d[i] * b.v;
  return r;
}
template <class S, int N>
__device__ __forceinline__ Dual<S, N> operator*(const Dual<S, N>& a, float s) {
  Dual<S, N> r;
  r.v = a.v * s;
#pragma unroll
  for (int i = 0; i < N; ++i) r.d[i] = a.d[i] * s;
  return r;
}
template <class S, int N>
__device__ __forceinline__ Dual<S, N> operator*(float s, const Dual<S, N>& a) { return a * s; }
template <class S, int N>
__device__ __forceinline__ Dual<S, N> operator+(const Dual<S, N>& a, float s) {
  Dual<S, N> r = a;
  r.v = a.v + s;
  return r;
}
template <class S, int N>
__device__ __forceinline__ Dual<S, N> operator-(const Dual<S, N>& a, float s) {
  Dual<S, N> r = a;
  r.v = a.v - s;
  return r;
}
template <class S, int N>
__device__ __forceinline__ Dual<S, N> operator-(float s, const Dual<S, N>& a) {
  return -(a - s);
}

// chain rule helper: f(a) with f(a.v) = fv and f'(a.v) = fd
template <class S, int N>
__device__ __forceinline__ Dual<S, N> chain(const Dual<S, N>& a, const S& fv, const S& fd) {
  Dual<S, N> r;
  r.v = fv;
#pragma unroll
  for (int i = 0; i < N; ++i) r.d[i] = fd * a.d[i];
  return r;
}

__device__ __forceinline__ float dsqrt(float a) { return sqrtf(a); }
__device__ __forceinline__ float drecip(float a) { return 1.0f / a; }
__device__ __forceinline__ float dsin(float a) { return sinf(a); }
__device__ __forceinline__ float dcos(float a) { return cosf(a); }
__device__ __forceinline__ float dexp(float a) { return expf(a); }

template <class S, int N>
__device__ __forceinline__ Dual<S, N> dsqrt(const Dual<S, N>& a) {
  S s = dsqrt(a.v);
  return chain(a, s, drecip(s) * 0.5f);
}
template <class S, int N>
__device__ __forceinline__ Dual<S, N> drecip(const Dual<S, N>& a) {
  S r = drecip(a.v);
  return chain(a, r, -(r * r));
}
template <class S, int N>
__device__ __forceinline__ Dual<S, N> dsin(const Dual<S, N>& a) {
  return chain(a, dsin(a.v), dcos(a.v));
}
template <class S, int N>
__device__ __forceinline__ Dual<S, N> dcos(const Dual<S, N>& a) {
  return chain(a, dcos(a.v), -dsin(a.v));
}
template <class S, int N>
__device__ __forceinline__ Dual<S, N> dexp(const Dual<S, N>& a) {
  S e = dexp(a.v);
  return chain(a, e, e);
}

// ---------------------------------------------------------------------------
// real spherical harmonics of one degree L, component normalisation
// ---------------------------------------------------------------------------
template <int L, class T>
__device__ __forceinline__ void sh_degree(const T& nx, const T& ny, const T& nz, T* Y) {
  if constexpr (L == 0) {
    Y[0] = T(1.f);
  } else if constexpr (L == 1) {
    const float c = 1.7320508075688772f;  // sqrt(3)
    Y[0] = ny * c;
    Y[1] = nz * c;
    Y[2] = nx * c;
  } else if constexpr (L == 2) {
    const float c15 = 3.872983346207417f;   // sqrt(15)
    const float c5h = 1.118033988749895f;   // sqrt(5)/2
    const float c15h = 1.9364916731037085f; // sqrt(15)/2
    Y[0] = (nx * ny) * c15;
    Y[1] = (ny * nz) * c15;
    Y[2] = ((nz * nz) * 3.f - 1.f) * c5h;
    Y[3] = (nx * nz) * c15;
    Y[4] = (nx * nx - ny * ny) * c15h;
  } else {
    const float a = 2.091650066335189f;   // sqrt(70)/4
    const float b = 10.246950765959598f;  // sqrt(105)
    const float c = 1.6201851746019651f;  // sqrt(42)/4
    const float d = 1.3228756555322954f;  // sqrt(7)/2
    const float e = 5.123475382979799f;   // sqrt(105)/2
    T x2 = nx * nx, y2 = ny * ny, z2 = nz * nz;
    T f = z2 * 5.f - 1.f;
    Y[0] = (ny * (x2 * 3.f - y2)) * a;
    Y[1] = (nx * ny * nz) * b;
    Y[2] = (ny * f) * c;
    Y[3] = (nz * (z2 * 5.f - 3.f)) * d;
    Y[4] = (nx * f) * c;
    Y[5] = (nz * (x2 - y2)) * e;
    Y[6] = (nx * (x2 - y2 * 3.f)) * a;
  }
}

template <class T>
__device__ __forceinline__ void unit(const T& x, const T& y, const T& z, T& nx, T& ny, T& nz, T& r) {
  r = dsqrt(x * x + y * y + z * z);
  T ri = drecip(r);
  nx = x * ri;
  ny = y * ri;
  nz = z * ri;
}

// all degrees 0..LMAX concatenated ((LMAX+1)^2 values)
template <int LMAX, class T>
__device__ __forceinline__ void sh_all(const T& nx, const T& ny, const T& nz, T* Y) {
  sh_degree<0>(nx, ny, nz, Y);
  if constexpr (LMAX >= 1) sh_degree<1>(nx, ny, nz, Y + 1);
  if constexpr (LMAX >= 2) sh_degree<2>(nx, ny, nz, Y + 4);
  if constexpr (LMAX >= 3) sh_degree<3>(nx, ny, nz, Y + 9);
}

// ---------------------------------------------------------------------------
// radial basis b_k(r), k < R (entries R..RM-1 are zero)
// ---------------------------------------------------------------------------
template <int RM, class T>
__device__ __forceinline__ void radial_basis(const DevPlan& pl, const T& r, T* b) {
  if (pl.radial == TPCONV_RADIAL_GAUSSIAN) {
#pragma unroll
    for (int k = 0; k < RM; ++k) {
      if (k < pl.R) {
        T t = (r - (pl.rp0 + float(k) * pl.rc0)) * pl.rc1;
        b[k] = dexp(-(t * t));
      } else {
        b[k] = T(0.f);
      }
    }
  } else {
    if (val(r) >= pl.rp0) {
#pragma unroll
      for (int k = 0; k < RM; ++k) b[k] = T(0.f);
      return;
    }
    T th = r * pl.rc0;                            // pi r / r_c
    T c1 = dcos(th), s1 = dsin(th);
    T fc = (c1 + 1.f) * 0.5f;                     // cosine cutoff (same angle)
    T pre = drecip(r) * fc * pl.rc1;              // sqrt(2/r_c) fc / r
    // sin((k+1) th) = 2 cos(th) sin(k th) - sin((k-1) th): one sin/cos pair per edge
    T c2 = c1 * 2.f;
    T sp = T(0.f), sk = s1;
#pragma unroll
    for (int k = 0; k < RM; ++k) {
      if (k < pl.R) b[k] = sk * pre;
      else b[k] = T(0.f);
      T sn = c2 * sk - sp;
      sp = sk;
      sk = sn;
    }
  }
}

// lane helpers
__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

template <int N>
__device__ __forceinline__ void warp_sum_all(float* v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
  }
}

#define TPC_FOR_EACH_TRIPLE(X)                                                                       \
  X(0, 0, 0) X(0, 1, 1) X(0, 2, 2) X(0, 3, 3) X(1, 0, 1) X(1, 1, 0) X(1, 1, 1) X(1, 1, 2) X(1, 2, 1) \
  X(1, 2, 2) X(1, 2, 3) X(1, 3, 2) X(1, 3, 3) X(2, 0, 2) X(2, 1, 1) X(2, 1, 2) X(2, 1, 3) X(2, 2, 0) \
  X(2, 2, 1) X(2, 2, 2) X(2, 2, 3) X(2, 3, 1) X(2, 3, 2) X(2, 3, 3) X(3, 0, 3) X(3, 1, 2) X(3, 1, 3) \
  X(3, 2, 1) X(3, 2, 2) X(3, 2, 3) X(3, 3, 0) X(3, 3, 1) X(3, 3, 2) X(3, 3, 3)

__host__ __device__ constexpr int triple_id(int a, int b, int c) { return a * 16 + b * 4 + c; }

}  // namespace tpc
