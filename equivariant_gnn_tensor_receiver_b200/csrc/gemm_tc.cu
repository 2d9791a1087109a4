// Tensor-core GEMM for the node-level Theta contraction (sm_100a: tcgen05 + TMEM + TMA).
//
//   C[m, n] (+)= sum_k A[m, k] B[n, k]       A: [M][K] fp32 row-major (K-major)
//                                            B: [N][K] fp32 row-major (K-major)
// C is written through a strided view, so rows (node, m) and columns (channel)
// land directly in the [node][mul][2l+1] feature layout.
//
// This is the mixing step of the streaming schedule ("Sobek", arXiv 2607.18074,
// abstract: fully connected multiplicity mixing applied to bounded receiver-side
// state): out_blk = A_blk . Theta_blk with A the receiver-side state.
//
// Precision modes:
//   TF32   one kind::tf32 MMA per K step (operands read as TF32).
//   3xTF32 fp32-accurate split (Ootomo & Yokota, 2022): a_hi = rn_tf32(a),
//          a_lo = rn_tf32(a - a_hi), both exactly representable in TF32;
//          C += A_hi B_hi + A_hi B_lo + A_lo B_hi.  Round-to-nearest (not
//          truncation) keeps the neglected terms uncorrelated with the sign of
//          a*b, so their sum grows like sqrt(K), not K.  The B split is
//          precomputed; the A split is done in shared memory by four converter
//          warps between the TMA load and the MMA.
//
// CTA: 6 warps.  warp 0 issues TMA loads (128 x 32 A tile and BN x 32 B tile,
// 128-byte swizzle) into a ring of shared-memory stages; warp 1 owns the TMEM
// accumulator (128 lanes x BN fp32 columns) and issues the MMAs from one thread;
// warps 2-5 split A (3xTF32) and run the epilogue (tcgen05.ld -> global).
// Every wait on the pipeline is bounded by the call's wait limit; on expiry the
// kernel records an error code and stops issuing work; before it exits it waits
// (bounded by a fixed limit) for its own loads and MMAs, then frees TMEM.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "gemm_tc.h"
#include "tc_common.cuh"

namespace tpc {

__device__ int g_tc_error;  // first error code recorded by a tensor-core GEMM (0 = none)

namespace {

using namespace tc;

constexpr int kBM = 128, kBK = 32;  // rows per CTA, fp32 K per stage (128 bytes)

// bounded wait on the kernel's own pipeline; on expiry records `code` and returns false
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, uint64_t limit, int code) {
  if (mbar_wait_for(b, parity, limit)) return true;
  atomicCAS(&g_tc_error, 0, code);
  return false;
}

// Column tiles of at most 64 run two CTAs per SM (two stages each: the same
// bytes in flight per SM as one CTA with four, in two independent pipelines,
// and twice the CTA slots for the partial waves); wider tiles one CTA.
template <int BN>
constexpr int tc_ctas_per_sm() {
  return BN <= 64 ? 2 : 1;
}

template <int BN>
struct TcSmem {
  static constexpr int kA = kBM * kBK * 4;   // 16 KB
  static constexpr int kB = BN * kBK * 4;    // BN x 128 B
  static constexpr int kStage = 2 * kA + 2 * kB;
  static constexpr int kStages = tc_ctas_per_sm<BN>() == 2
                                     ? 2
                                     : ((200 * 1024) / kStage >= 4 ? 4 : ((200 * 1024) / kStage >= 3 ? 3 : 2));
  static constexpr int kBytes = kStages * kStage + 1024 /*align*/ + 256 /*barriers: 3 x stages + 5, slot, flag*/;
};

// Accumulators in TMEM.  The 3xTF32 mode uses NACC of them in the round
// schedule of tc_common.cuh (chains of 4 K steps, rounds added into fp32
// registers), for column tiles of at most 128; with 256 columns (only used for
// short K) the K steps alternate over two accumulators summed at the end.
template <int BN, bool SPLIT>
struct TcAcc {
  static constexpr int kCols = BN < 32 ? 32 : BN;
  // TMEM columns of one CTA: 512 / (CTAs per SM)
  static constexpr int kMaxCols = 512 / tc_ctas_per_sm<BN>();
  static constexpr int N = SPLIT ? (kMaxCols / kCols > 8 ? 8 : kMaxCols / kCols) : 1;
  static constexpr uint32_t kAlloc = kCols * N;  // power of two, <= 512
  static constexpr bool kDrain = SPLIT && BN <= 128;
};

template <int BN, bool SPLIT>
__global__ void __launch_bounds__(192, tc_ctas_per_sm<BN>())
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmBlo, const __grid_constant__ CUtensorMap tmC, int M, int N,
              int K, TcOut out, int accumulate, int tma_out, uint64_t limit) {
  using SM = TcSmem<BN>;
  constexpr int S = SM::kStages;
  constexpr uint32_t kCols = TcAcc<BN, SPLIT>::kCols;
  constexpr int NACC = TcAcc<BN, SPLIT>::N;
  constexpr uint32_t kAlloc = TcAcc<BN, SPLIT>::kAlloc;
  constexpr bool DRAIN = TcAcc<BN, SPLIT>::kDrain;
  using RS = Rounds<NACC>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + S * SM::kStage);
  uint64_t* conv = full + S;
  uint64_t* empty = conv + S;
  uint64_t* accf = empty + S;
  uint64_t* bfull = accf + 1;  // [2] a round of the bank is complete (round schedule)
  uint64_t* bfree = bfull + 2; // [2] the bank has been added into registers
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bfree + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kBM;
  const int n0 = blockIdx.y * BN;
  const int nk = (K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&conv[s], 128);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bfull[b], 1);
      mbar_init(&bfree[b], 128);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(tmem_slot, kAlloc);
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  auto sA = [&](int s) { return base + s * SM::kStage; };
  auto sAlo = [&](int s) { return base + s * SM::kStage + SM::kA; };
  auto sB = [&](int s) { return base + s * SM::kStage + 2 * SM::kA; };
  auto sBlo = [&](int s) { return base + s * SM::kStage + 2 * SM::kA + SM::kB; };

  int issued = 0;  // TMA stages issued by warp 0
  if (warp == 0) {
    if (lane == 0) {
      const uint32_t bytes = SM::kA + (SPLIT ? 2 : 1) * SM::kB;
      for (int kt = 0; kt < nk; ++kt) {
        const int s = kt % S;
        if (kt >= S && !mbar_wait(&empty[s], ((kt / S) + 1) & 1, limit, 1)) {
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        mbar_expect_tx(&full[s], bytes);
        tma_load_2d(sA(s), &tmA, &full[s], kt * kBK, m0);
        tma_load_2d(sB(s), &tmB, &full[s], kt * kBK, n0);
        if (SPLIT) tma_load_2d(sBlo(s), &tmBlo, &full[s], kt * kBK, n0);
        issued = kt + 1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_tf32(kBM, BN);
      for (int kt = 0; kt < nk; ++kt) {
        const int s = kt % S;
        const uint32_t par = (kt / S) & 1;
        // round schedule: round r = kt / D writes bank r & 1, free again once round r - 2 was drained
        const int r = DRAIN ? kt / RS::D : 0, j = DRAIN ? kt - r * RS::D : kt, bank = r & 1;
        if (DRAIN && j == 0 && r >= 2 && !mbar_wait(&bfree[bank], ((r >> 1) - 1) & 1, limit, 7)) {
          *abort_flag = 1;
          break;
        }
        if (!mbar_wait(SPLIT ? &conv[s] : &full[s], par, limit, 2) || *abort_flag) {
          *abort_flag = 1;
          break;
        }
        fence_after_sync();
        const uint32_t a = smem_u32(sA(s)), al = smem_u32(sAlo(s)), b = smem_u32(sB(s)), bl = smem_u32(sBlo(s));
        const int ai = DRAIN ? bank * RS::NPB + j % RS::NPB : kt % NACC;
        const int fresh = DRAIN ? RS::NPB : NACC;  // the first `fresh` steps of a round (of the call) overwrite
        const uint32_t td = tmem + uint32_t(ai * kCols);
#pragma unroll
        for (int kk = 0; kk < kBK / 8; ++kk) {
          const uint32_t off = kk * 32;  // 8 TF32 = 32 bytes along K inside the swizzle atom
          const uint32_t acc = (j >= fresh || kk > 0) ? 1u : 0u;
          mma_tf32(td, sw128_kmajor(a + off), sw128_kmajor(b + off), idesc, acc);
          if (SPLIT) {
            mma_tf32(td, sw128_kmajor(a + off), sw128_kmajor(bl + off), idesc, 1u);
            mma_tf32(td, sw128_kmajor(al + off), sw128_kmajor(b + off), idesc, 1u);
          }
        }
        mma_commit(&empty[s]);
        if (DRAIN && (j == RS::D - 1 || kt == nk - 1)) mma_commit(&bfull[bank]);
      }
      mma_commit(accf);
    }
  } else {
    // warps 2..5: split A in shared memory (3xTF32), add finished rounds of
    // accumulators into registers, then the epilogue
    const int t = threadIdx.x - 64;  // 0..127
    const int q = warp & 3;          // TMEM lane quadrant this warp may access
    const uint32_t tlane = tmem + (uint32_t(q * 32) << 16);
    constexpr int NR = DRAIN ? BN : 16;  // register accumulators (unused without the round schedule)
    float racc[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) racc[i] = 0.f;
    int drained = 0;  // rounds added into racc
    // every exit decision of these warps is made warp-uniform (__all_sync): the
    // TMEM loads below are warp-collective
    auto drain = [&](int rr) -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(&bfull[rr & 1], (rr >> 1) & 1, limit, 8))) return false;
      fence_after_sync();
      tmem_drain<NR, RS::NPB>(tlane, rr & 1, min(RS::NPB, RS::steps(rr, nk)), kCols, racc);
      fence_before_sync();
      mbar_arrive(&bfree[rr & 1]);
      ++drained;
      return true;
    };
    if (SPLIT) {
      for (int kt = 0; kt < nk; ++kt) {
        const int s = kt % S;
        if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (kt / S) & 1, limit, 3) && !*abort_flag)) {
          *abort_flag = 1;
          break;
        }
        float4* a4 = reinterpret_cast<float4*>(sA(s));
        float4* l4 = reinterpret_cast<float4*>(sAlo(s));
#pragma unroll 4
        for (int i = t; i < kBM * kBK / 4; i += 128) split4(a4 + i, l4 + i);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(&conv[s]);
        if constexpr (DRAIN) {
          const int rr = RS::drain_after(kt);
          if (rr >= 0 && !drain(rr)) {
            *abort_flag = 1;
            break;
          }
        }
      }
    }
    bool ok = __all_sync(0xffffffffu, mbar_wait(accf, 0, limit, 4) && !*abort_flag);
    fence_after_sync();
    if constexpr (DRAIN) {
      const int nrounds = (nk + RS::D - 1) / RS::D;
      while (ok && drained < nrounds) ok = drain(drained);
    }
    // plain row-major output (tma_out): the tile goes through the operand ring,
    // idle once every MMA has completed, as BN / 32 boxes of 128 rows x 128 bytes
    // in the 128-byte swizzle, and leaves by TMA stores
    if (tma_out && !ok) *abort_flag = 1;
    if (ok && tma_out) {
      const int r = q * 32 + lane;
      const int nacc = nk < NACC ? nk : NACC;
#pragma unroll
      for (int c = 0; c < BN; c += 16) {
        float v[16];
        if constexpr (DRAIN) {
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = racc[(c + i) % NR];
        } else {
          tmem_ld16(tlane + uint32_t(c), v);
          for (int a = 1; a < nacc; ++a) {
            float w[16];
            tmem_ld16(tlane + uint32_t(a * kCols + c), w);
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] += w[i];
          }
        }
        float* box = reinterpret_cast<float*>(base + (c / 32) * (kBM * 128));
        const int j0 = (c % 32) / 4;  // first 16-byte chunk of these 16 columns in the box row
#pragma unroll
        for (int i = 0; i < 4; ++i)
          *reinterpret_cast<float4*>(box + r * 32 + (((j0 + i) ^ (r & 7)) * 4)) =
              make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      }
    } else if (ok) {
      const int row = m0 + q * 32 + lane;
      const int64_t rbase = (row / out.rdiv) * out.r_hi + (row % out.rdiv) * out.r_lo;
      const int nacc = nk < NACC ? nk : NACC;  // accumulators that received a K step
#pragma unroll
      for (int c = 0; c < BN; c += 16) {
        float v[16];
        if constexpr (DRAIN) {
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = racc[(c + i) % NR];
        } else {
          tmem_ld16(tlane + uint32_t(c), v);
          for (int a = 1; a < nacc; ++a) {
            float w[16];
            tmem_ld16(tlane + uint32_t(a * kCols + c), w);
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] += w[i];
          }
        }
        if (row < M) {
          float* dst0 = out.p + rbase + int64_t(n0 + c) * out.c_hi;
          if (out.c_hi == 1 && n0 + c + 16 <= N && (reinterpret_cast<uintptr_t>(dst0) & 15) == 0) {
            float4* d4 = reinterpret_cast<float4*>(dst0);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float4 t = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
              if (accumulate) {
                const float4 o = d4[i];
                t.x += o.x;
                t.y += o.y;
                t.z += o.z;
                t.w += o.w;
              }
              d4[i] = t;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int col = n0 + c + i;
              if (col < N) {
                float* dst = out.p + rbase + int64_t(col) * out.c_hi;
                *dst = accumulate ? *dst + v[i] : v[i];
              }
            }
          }
        }
      }
    }
  }
  if (tma_out && warp >= 2) {
    // every epilogue thread's writes are visible to the async proxy before one
    // thread stores the boxes; all four warps pass the barrier whatever happened
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (threadIdx.x == 64 && !*abort_flag) {
#pragma unroll 1
      for (int b = 0; b < BN / 32; ++b) tma_store_2d(&tmC, base + b * (kBM * 128), n0 + 32 * b, m0);
      tma_store_commit_and_wait_read();  // the boxes stay in shared memory until read
    }
  }
  // drain: the producer waits (bounded) for the loads it issued so no copy is
  // in flight when the CTA exits, then TMEM is released
  if (warp == 0 && lane == 0 && *abort_flag) {
    for (int kt = (issued > S ? issued - S : 0); kt < issued; ++kt)
      mbar_wait(&full[kt % S], (kt / S) & 1, kDrainLimitNs, 5);
  }
  // the MMA thread waits for its own MMAs before TMEM is released
  if (warp == 1 && lane == 0) mbar_wait(accf, 0, kDrainLimitNs, 6);
  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    tmem_dealloc(tmem, kAlloc);
  }
}

// ---- host side ---------------------------------------------------------------
using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encoder() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  return fn;
}

// rows x cols fp32 row-major with leading dimension ld (elements); box box_rows x 32
bool make_map(CUtensorMap* m, const float* p, int64_t rows, int64_t cols, int64_t ld, int box_rows) {
  EncodeFn enc = encoder();
  if (!enc) return false;
  if ((reinterpret_cast<uintptr_t>(p) & 15) || ((ld * 4) & 15) || rows <= 0 || cols <= 0) return false;
  cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(ld * 4)};
  cuuint32_t box[2] = {cuuint32_t(kBK), cuuint32_t(box_rows)};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(p), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, bool SPLIT>
cudaError_t run(const float* A, int64_t lda, const float* B, const float* Blo, int64_t ldb, int M, int N, int K,
                TcOut out, int accumulate, uint64_t limit, cudaStream_t st) {
  CUtensorMap ta, tb, tbl, tc;
  if (!make_map(&ta, A, M, K, lda, kBM) || !make_map(&tb, B, N, K, ldb, BN)) return cudaErrorInvalidValue;
  if (SPLIT && !make_map(&tbl, Blo, N, K, ldb, BN)) return cudaErrorInvalidValue;
  if (!SPLIT) tbl = tb;
  // a plain row-major output C[i][j] = p[i * r_hi + j], written (not added), leaves by TMA stores
  const int tma_out = !accumulate && out.rdiv == 1 && out.r_lo == 0 && out.c_hi == 1 &&
                      make_map(&tc, out.p, M, N, out.r_hi, kBM);
  if (!tma_out) tc = ta;
  using SM = TcSmem<BN>;
  static_assert(BN / 32 * kBM * 128 <= SM::kStages * SM::kStage, "the output tile fits the operand ring");
  dim3 grid(unsigned((M + kBM - 1) / kBM), unsigned((N + BN - 1) / BN));
  k_gemm_tc<BN, SPLIT><<<grid, 192, SM::kBytes, st>>>(ta, tb, tbl, tc, M, N, K, out, accumulate, tma_out, limit);
  return cudaGetLastError();
}

template <int BN, bool SPLIT>
cudaError_t set_smem() {
  return cudaFuncSetAttribute(k_gemm_tc<BN, SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcSmem<BN>::kBytes);
}

}  // namespace

cudaError_t gemm_tc_init() {
  cudaError_t e = cudaSuccess;
  for (cudaError_t r : {set_smem<32, true>(), set_smem<64, true>(), set_smem<128, true>(), set_smem<256, true>(),
                        set_smem<32, false>(), set_smem<64, false>(), set_smem<128, false>(), set_smem<256, false>()})
    if (r != cudaSuccess && e == cudaSuccess) e = r;
  return e;
}

bool gemm_tc_supported(const float* A, int64_t lda, const float* B, int64_t ldb, int M, int N, int K) {
  if (!encoder()) return false;
  if (M <= 0 || N <= 0 || K <= 0) return false;
  if ((reinterpret_cast<uintptr_t>(A) & 15) || (reinterpret_cast<uintptr_t>(B) & 15)) return false;
  if ((lda & 3) || (ldb & 3)) return false;
  return true;
}

cudaError_t gemm_tc(const float* A, int64_t lda, const float* B, const float* Blo, int64_t ldb, int M, int N, int K,
                    TcOut out, int accumulate, bool split, cudaStream_t st, uint64_t limit) {
  // 3xTF32 with long K uses column tiles of at most 128, whose accumulators are
  // drained into registers in rounds (bounded TMEM accumulation chains)
  const int bn = N <= 32 ? 32 : (N <= 64 ? 64 : ((N <= 128 || (split && K > 256)) ? 128 : 256));
  if (split) {
    switch (bn) {
      case 32: return run<32, true>(A, lda, B, Blo, ldb, M, N, K, out, accumulate, limit, st);
      case 64: return run<64, true>(A, lda, B, Blo, ldb, M, N, K, out, accumulate, limit, st);
      case 128: return run<128, true>(A, lda, B, Blo, ldb, M, N, K, out, accumulate, limit, st);
      default: return run<256, true>(A, lda, B, Blo, ldb, M, N, K, out, accumulate, limit, st);
    }
  }
  switch (bn) {
    case 32: return run<32, false>(A, lda, B, Blo, ldb, M, N, K, out, accumulate, limit, st);
    case 64: return run<64, false>(A, lda, B, Blo, ldb, M, N, K, out, accumulate, limit, st);
    case 128: return run<128, false>(A, lda, B, Blo, ldb, M, N, K, out, accumulate, limit, st);
    default: return run<256, false>(A, lda, B, Blo, ldb, M, N, K, out, accumulate, limit, st);
  }
}

cudaError_t gemm_tc_read_error(int* code) {
  int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(code, g_tc_error, sizeof(int));
  if (e) return e;
  return *code ? cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(int)) : cudaSuccess;
}

// Theta^T split: hi[n][k] = rn_tf32(Theta[k][n]), lo = rn_tf32(Theta - hi)
__global__ void k_split_transpose(const float* __restrict__ th, int K, int N, float* __restrict__ hi,
                                  float* __restrict__ lo) {
  __shared__ float tile[32][33];
  const int k0 = blockIdx.x * 32, n0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int k = k0 + i, n = n0 + threadIdx.x;
    tile[i][threadIdx.x] = (k < K && n < N) ? th[int64_t(k) * N + n] : 0.f;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int n = n0 + i, k = k0 + threadIdx.x;
    if (n < N && k < K) {
      const float v = tile[threadIdx.x][i];
      const float h = rn_tf32(v);
      if (lo) {
        hi[int64_t(n) * K + k] = h;
        lo[int64_t(n) * K + k] = rn_tf32(v - h);
      } else {
        hi[int64_t(n) * K + k] = v;
      }
    }
  }
}

cudaError_t split_transpose(const float* th, int K, int N, float* hi, float* lo, cudaStream_t st) {
  dim3 grid(unsigned((K + 31) / 32), unsigned((N + 31) / 32));
  k_split_transpose<<<grid, dim3(32, 8), 0, st>>>(th, K, N, hi, lo);
  return cudaGetLastError();
}

// elementwise split: hi = rn_tf32(v), lo = rn_tf32(v - hi)  (lo may be null: hi = v)
__global__ void k_split(const float* __restrict__ v, int64_t n, float* __restrict__ hi, float* __restrict__ lo) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const float a = v[i];
    if (lo) {
      const float h = rn_tf32(a);
      hi[i] = h;
      lo[i] = rn_tf32(a - h);
    } else {
      hi[i] = a;
    }
  }
}

cudaError_t split_elementwise(const float* v, int64_t n, float* hi, float* lo, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const int blocks = int(std::min<int64_t>((n + 255) / 256, 148 * 8));
  k_split<<<blocks, 256, 0, st>>>(v, n, hi, lo);
  return cudaGetLastError();
}

// Theta of each path as [c_in][K_x] of its input block, column kxoff(p) + k*c_out + w
// (dx = B . Theta operand); optional TF32 split.  blockIdx.y = path of the list; the
// blocks along x stride over its R c_in c_out entries.
__global__ void k_theta_x_all(const float* __restrict__ th, const __grid_constant__ XPackList l,
                              float* __restrict__ hi, float* __restrict__ lo) {
  const XPackPath& q = l.p[blockIdx.y];
  const int64_t n = int64_t(l.R) * q.c_in * q.c_out;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const int w = int(i % q.c_out);
    const int64_t t = i / q.c_out;
    const int u = int(t % q.c_in), k = int(t / q.c_in);
    const float a = th[q.theta_off + i];  // Theta[p][k][u][w]
    const int64_t o = q.dst_off + int64_t(u) * q.Kx + q.kxoff + int64_t(k) * q.c_out + w;
    if (lo) {
      const float h = rn_tf32(a);
      hi[o] = h;
      lo[o] = rn_tf32(a - h);
    } else {
      hi[o] = a;
    }
  }
}

cudaError_t theta_x_pack_all(const float* th, const XPackList& l, float* hi, float* lo, cudaStream_t st) {
  if (l.n <= 0 || l.n > kXPackMax) return l.n == 0 ? cudaSuccess : cudaErrorInvalidValue;
  int64_t nmax = 0;
  for (int i = 0; i < l.n; ++i) nmax = std::max<int64_t>(nmax, int64_t(l.R) * l.p[i].c_in * l.p[i].c_out);
  if (nmax <= 0) return cudaSuccess;
  const int bx = int(std::min<int64_t>((nmax + 255) / 256, std::max(1, 148 * 8 / l.n)));
  k_theta_x_all<<<dim3(unsigned(bx), unsigned(l.n)), 256, 0, st>>>(th, l, hi, lo);
  return cudaGetLastError();
}

// g block of output block (offset, mul, 2l+1) of nodes r0 : r0+nc as [(node, m)][w]
__global__ void k_pack_rows(const float* __restrict__ g, int dim, int off, int mul, int n3, int64_t r0, int nc,
                            float* __restrict__ out) {
  const int64_t total = int64_t(nc) * n3 * mul;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
    const int w = int(i % mul);
    const int64_t rm = i / mul;
    const int m = int(rm % n3);
    const int64_t r = rm / n3;
    out[i] = g[(r0 + r) * dim + off + int64_t(w) * n3 + m];
  }
}

cudaError_t pack_rows(const float* g, int dim, int off, int mul, int n3, int64_t r0, int nc, float* out,
                      cudaStream_t st) {
  const int64_t total = int64_t(nc) * n3 * mul;
  if (total <= 0) return cudaSuccess;
  const int blocks = int(std::min<int64_t>((total + 255) / 256, 148 * 16));
  k_pack_rows<<<blocks, 256, 0, st>>>(g, dim, off, mul, n3, r0, nc, out);
  return cudaGetLastError();
}

}  // namespace tpc
