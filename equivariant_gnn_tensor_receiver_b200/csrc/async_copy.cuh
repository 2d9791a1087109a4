// Asynchronous global -> shared copies (cp.async) used to stage gathered rows.
#pragma once

#include <stdint.h>

namespace tpc {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// 4-byte copy through L1
__device__ __forceinline__ void ac_copy4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
// 16-byte copy through L1 (both addresses 16-byte aligned)
__device__ __forceinline__ void ac_copy16(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void ac_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// wait until at most N of this thread's committed groups are still in flight
template <int N>
__device__ __forceinline__ void ac_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float4 lds4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void sts4(float* p, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}

// load N (multiple of 4) consecutive floats from 16-byte aligned shared memory
template <int N>
__device__ __forceinline__ void lds_vec(const float* p, float* v) {
  static_assert(N % 4 == 0, "vector width");
#pragma unroll
  for (int i = 0; i < N / 4; ++i) {
    const float4 t = lds4(p + 4 * i);
    v[4 * i] = t.x;
    v[4 * i + 1] = t.y;
    v[4 * i + 2] = t.z;
    v[4 * i + 3] = t.w;
  }
}
// load NP (even) consecutive float pairs from 16-byte aligned shared memory
template <int NP>
__device__ __forceinline__ void lds_f2(const float* p, float2* v) {
  static_assert(NP % 2 == 0, "pairs come in 16-byte groups");
#pragma unroll
  for (int i = 0; i < NP / 2; ++i) {
    const float4 t = lds4(p + 4 * i);
    v[2 * i] = make_float2(t.x, t.y);
    v[2 * i + 1] = make_float2(t.z, t.w);
  }
}
template <int N>
__device__ __forceinline__ void sts_vec(float* p, const float* v) {
  static_assert(N % 4 == 0, "vector width");
#pragma unroll
  for (int i = 0; i < N / 4; ++i) sts4(p + 4 * i, v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}

}  // namespace tpc
