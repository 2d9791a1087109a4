// Device helpers of the tensor-core kernels (sm_100a): mbarriers with bounded
// waits, TMA tile loads, shared-memory matrix descriptors (128-byte swizzle),
// the kind::tf32 instruction descriptor, tcgen05.mma / commit / ld, and the
// round-to-nearest TF32 split of the 3xTF32 method (Ootomo & Yokota, 2022).
//
// Field layouts follow the PTX ISA's definitions of the tcgen05 shared-memory
// descriptor and instruction descriptor (an interface, written out here).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tpc {
namespace tc {

constexpr uint64_t kDrainLimitNs = 2000000000ull;  // waits for a CTA's own copies / MMAs before it exits

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase with the given parity to complete, for at most limit_ns of
// %globaltimer.  Returns false when the limit expires (nothing is recorded here).
__device__ __forceinline__ bool mbar_wait_for(uint64_t* b, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try(b, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try(b, parity)) {
    if (global_ns() - t0 > limit_ns) return false;
  }
  return true;
}

__device__ __forceinline__ float rn_tf32(float a) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(a));
  return __uint_as_float(r);
}

// 2-D tiled TMA load into shared memory, completion counted on an mbarrier (no multicast)
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// 2-D tiled TMA store of a shared-memory box (bulk async group of this thread);
// elements outside the tensor are not written
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void tma_store_commit_and_wait_read() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle: start address >> 4 in
// [0,14), leading byte offset >> 4 in [16,30), stride byte offset >> 4 in
// [32,46), version 1 at [46,48), layout SWIZZLE_128B = 2 at [61,64).
//   K-major operand : 8-row x 128-byte atoms stacked along the rows (SBO = 1024);
//                     the leading offset is unused.
//   (MN-major TF32 operands need the 32-byte-atom variant below.)
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFF) >> 4);
  d |= uint64_t((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= uint64_t((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}
__device__ __forceinline__ uint64_t sw128_kmajor(uint32_t saddr) { return sw128_desc(saddr, 16, 1024); }

// MN-major TF32 operands take the one layout the tensor core accepts for them:
// the 128-byte swizzle with 32-byte atomicity (layout type 1 at [61,64); TMA's
// CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B writes it).  Atoms of 4 K-rows x 128 bytes
// (32 fp32 along M / N), the 32-byte pieces of a row permuted by the row index
// mod 4.  LBO = bytes between atoms along M / N, SBO = bytes between 4-row
// groups along K.
__device__ __forceinline__ uint64_t sw128b32_mn_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFF) >> 4);
  d |= uint64_t((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= uint64_t((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(1) << 61;
  return d;
}

// Instruction descriptor of kind::tf32 with fp32 accumulation: D format F32 at
// [4,6), A and B format TF32 at [7,10) and [10,13), A / B major-ness at bits 15
// / 16 (0 = K-major, 1 = MN-major), N >> 3 at [17,23), M >> 4 at [24,29).
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, bool a_mn = false, bool b_mn = false) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (a_mn ? 1u << 15 : 0u) | (b_mn ? 1u << 16 : 0u) |
         (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
// arrive on the mbarrier once every MMA issued so far by this thread has completed
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 16 consecutive fp32 columns of the warp's 32 TMEM lanes (one per thread)
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(cols));
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols));
}
__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;"); }

// 3xTF32 split of a float4 in shared memory: a = hi (in place), lo = remainder
__device__ __forceinline__ void split4(float4* a, float4* lo) {
  const float4 v = *a;
  float4 h, l;
  h.x = rn_tf32(v.x);
  h.y = rn_tf32(v.y);
  h.z = rn_tf32(v.z);
  h.w = rn_tf32(v.w);
  l.x = rn_tf32(v.x - h.x);
  l.y = rn_tf32(v.y - h.y);
  l.z = rn_tf32(v.z - h.z);
  l.w = rn_tf32(v.w - h.w);
  *a = h;
  *lo = l;
}

// ---- accumulation schedule of the 3xTF32 kernels ------------------------------
// The tensor core accumulates in fp32 inside TMEM; its rounding error grows with
// the length of an accumulation chain, i.e. with K.  The NACC accumulators form
// two banks of NPB.  K steps run in rounds of D = 4 NPB steps; round r writes
// bank r & 1, each accumulator starting afresh and taking every NPB-th step, so
// no chain is longer than 4 K steps (48 MMAs of K = 8).  The epilogue warps add
// a finished round's bank into fp32 registers (round to nearest) halfway through
// the next round and release the bank for round r + 2; a round's last MMA
// commits to bank_full, the drain arrives on bank_free.
template <int NACC>
struct Rounds {
  static constexpr int NPB = NACC / 2;  // accumulators per bank
  static constexpr int D = 4 * NPB;     // K steps per round
  __device__ static int steps(int r, int nk) { return min(D, nk - r * D); }
  // the converter / epilogue warps drain round r right after handling K step kt, or -1
  __device__ static int drain_after(int kt) {
    const int t = kt + 1 - D / 2;
    return (t >= D && t % D == 0) ? t / D - 1 : -1;
  }
};

// add the accumulators of one bank that a round wrote (n_used <= NPB, warp-uniform)
// into racc; tlane = TMEM address of this warp's lane quadrant, column 0
template <int BN, int NPB>
__device__ __forceinline__ void tmem_drain(uint32_t tlane, int bank, int n_used, uint32_t cols, float (&racc)[BN]) {
#pragma unroll
  for (int c = 0; c < BN; c += 16) {
#pragma unroll
    for (int a = 0; a < NPB; ++a) {
      if (a < n_used) {
        float w[16];
        tmem_ld16(tlane + uint32_t((bank * NPB + a) * cols + c), w);
#pragma unroll
        for (int i = 0; i < 16; ++i) racc[c + i] += w[i];
      }
    }
  }
}

}  // namespace tc
}  // namespace tpc
