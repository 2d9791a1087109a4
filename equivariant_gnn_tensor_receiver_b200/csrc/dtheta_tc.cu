// Theta gradient on the tensor cores (tcgen05 + TMEM + TMA), deterministic split-K.
//
// For every path p (input block i1) and each operand pair (x, B) of a call
// (one pair in the backward, (x, B1) and (gg_x, B0) in the double backward):
//
//     dTheta[p][k][u][w] += sum_{s in chunk} sum_m1 x[s, u, m1] B[(s, m1), kxoff(p) + k c_out + w]
//
// the dense contraction of the Theta gradient that the mixing of "Sobek"
// (arXiv 2607.18074, abstract: fully connected multiplicity mixing) leaves
// behind.  Per path it is a GEMM with rows (k, w) (M = R c_out), columns u
// (N = c_in) and the reduction over K = (node, m1) (nc (2 l1 + 1) rows):
//
//     D[(k, w)][u] = sum_K Bs[K][(k, w)] Xt[u][K]
//
//   A operand = the sender-side state B, read in place.  Along a row of B the
//               (k, w) columns are contiguous, so A is "MN-major": TMA loads
//               32 (M) x 32 (K) boxes, four per 128-row tile, in the layout
//               the tensor core takes for MN-major TF32 operands (128-byte
//               swizzle with 32-byte atomicity: atoms of 4 K-rows x 128 bytes;
//               4096 bytes between atoms along M, 512 along K).
//   B operand = Xt[u][K], x of the chunk transposed per input block (K-major),
//               packed by k_pack_xt (already split into TF32 hi / lo).
//
// Work: every (pair, path) group has ceil(M / 128) row tiles, each split over
// K into ranges of kc rows (a multiple of 32); one CTA per (tile, range) keeps
// its 128 x BN fp32 partial in TMEM and stores it to a partial buffer.
// k_dtheta_reduce then adds the partials of a tile to dTheta in a fixed order
// (pair, range): no atomics, so the result is bitwise reproducible.
//
// Precision: 3xTF32 (a_hi b_hi + a_hi b_lo + a_lo b_hi, round-to-nearest
// splits, Ootomo & Yokota 2022), with the K steps of a CTA spread over several
// TMEM accumulators summed in fp32 at the end; or one TF32 pass.
//
// CTA: 6 warps.  Warp 0 issues the TMA loads, warp 1 owns TMEM and issues the
// MMAs from one thread, warps 2-5 split the A tile (3xTF32) and store the
// partial tile.  Data waits give up after the call's wait limit and record an
// error code; before exiting, a CTA waits (bounded by a fixed limit) for its
// own copies and MMAs, then frees TMEM.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "dtheta_tc.h"
#include "tc_common.cuh"

namespace tpc {

__device__ int g_dt_error;  // first error code recorded by a wait of k_dtheta_tc (0 = none)

namespace {

using namespace tc;

constexpr int kBM = 128, kBK = 32;
constexpr int kMaxMaps = 2 * kMaxBlocks;   // (pair, input block)
constexpr int kMaxGroups = 2 * kMaxPaths;  // (pair, path)
constexpr int kMaxSms = 160;               // partial buffer: two tiles per SM on up to this many SMs

int64_t sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev))
    return 148;
  return std::min(n, kMaxSms);
}

struct DtGroup {
  int cta0;    // first CTA of the group
  int n_mt;    // 128-row tiles (M = R c_out)
  int n_split; // K ranges per tile
  int kc;      // K rows per range (multiple of 32)
  int K;       // nc (2 l1 + 1)
  int a_col;   // column of the path's (k = 0, w = 0) in its B block
  int map;     // operand maps of (pair, i1)
};

struct __align__(64) DtParams {
  CUtensorMap a[kMaxMaps];   // B state [K][Kx] of (pair, i1), box 32 x 32, 128-byte swizzle, 32-byte atoms
  CUtensorMap bh[kMaxMaps];  // Xt hi [c_in][K], box 32 x BN, SW128
  CUtensorMap bl[kMaxMaps];  // Xt lo (3xTF32 only)
  DtGroup g[kMaxGroups];
  int n_groups;
  float* partial;            // [cta][BN][128]
  uint64_t wait_ns;
};

// Column tiles of at most 64 run two CTAs per SM (two stages and four TMEM
// accumulators each), wider tiles one; the planner sizes the split for that.
constexpr int dt_ctas_per_sm(int bn) { return bn <= 64 ? 2 : 1; }

template <int BN>
struct DtSmem {
  static constexpr int kA = kBM * kBK * 4;  // 16 KB: four 32 x 32 boxes
  static constexpr int kB = BN * kBK * 4;
  static constexpr int kStage = 2 * kA + 2 * kB;
  static constexpr int kStages = dt_ctas_per_sm(BN) == 2
                                     ? 2
                                     : ((200 * 1024) / kStage >= 4 ? 4 : ((200 * 1024) / kStage >= 3 ? 3 : 2));
  static constexpr int kBytes = kStages * kStage + 1024 + 256;
};

// TMEM accumulators; 3xTF32 with column tiles of at most 128 runs the round
// schedule of tc_common.cuh (accumulation chains of 4 K steps, rounds added
// into fp32 registers), which keeps fp32 accuracy for the long K of this GEMM.
template <int BN, bool SPLIT>
struct DtAcc {
  static constexpr int kCols = BN < 32 ? 32 : BN;
  static constexpr int kMaxCols = 512 / dt_ctas_per_sm(BN);  // TMEM columns of one CTA
  static constexpr int N = SPLIT ? (kMaxCols / kCols > 8 ? 8 : kMaxCols / kCols) : 1;
  static constexpr uint32_t kAlloc = kCols * N;
  static constexpr bool kDrain = SPLIT && BN <= 128;
};

// record the first error of the launch and report expiry
__device__ __forceinline__ bool waitp(uint64_t* b, uint32_t parity, uint64_t limit, int code) {
  if (mbar_wait_for(b, parity, limit)) return true;
  atomicCAS(&g_dt_error, 0, code);
  return false;
}

template <int BN, bool SPLIT>
__global__ void __launch_bounds__(192, dt_ctas_per_sm(BN)) k_dtheta_tc(const __grid_constant__ DtParams P) {
  using SM = DtSmem<BN>;
  constexpr int S = SM::kStages;
  constexpr uint32_t kCols = DtAcc<BN, SPLIT>::kCols;
  constexpr int NACC = DtAcc<BN, SPLIT>::N;
  constexpr uint32_t kAlloc = DtAcc<BN, SPLIT>::kAlloc;
  constexpr bool DRAIN = DtAcc<BN, SPLIT>::kDrain;
  using RS = Rounds<NACC>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + S * SM::kStage);
  uint64_t* conv = full + S;
  uint64_t* empty = conv + S;
  uint64_t* accf = empty + S;
  uint64_t* bfull = accf + 1;   // [2] a round of the bank is complete
  uint64_t* bfree = bfull + 2;  // [2] the bank has been added into registers
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bfree + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's group, row tile and K range
  int gi = 0;
  for (int i = 1; i < P.n_groups; ++i)
    if (P.g[i].cta0 <= int(blockIdx.x)) gi = i;
  const DtGroup& G = P.g[gi];
  const int local = int(blockIdx.x) - G.cta0;
  const int mt = local / G.n_split, sp = local - mt * G.n_split;
  const int k0 = sp * G.kc;
  const int k1 = min(G.K, k0 + G.kc);
  const int nk = k1 > k0 ? (k1 - k0 + kBK - 1) / kBK : 0;
  const int mcol = G.a_col + mt * kBM;
  const uint64_t limit = P.wait_ns;

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

  int issued = 0;
  if (warp == 0) {
    if (lane == 0) {
      const uint32_t bytes = SM::kA + (SPLIT ? 2 : 1) * SM::kB;
      const CUtensorMap* ma = &P.a[G.map];
      const CUtensorMap* mbh = &P.bh[G.map];
      const CUtensorMap* mbl = &P.bl[G.map];
      for (int kt = 0; kt < nk; ++kt) {
        const int s = kt % S;
        if (kt >= S && !waitp(&empty[s], ((kt / S) + 1) & 1, limit, 1)) {
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        const int kr = k0 + kt * kBK;
        mbar_expect_tx(&full[s], bytes);
#pragma unroll
        for (int j = 0; j < kBM / 32; ++j) tma_load_2d(sA(s) + j * 4096, ma, &full[s], mcol + 32 * j, kr);
        tma_load_2d(sB(s), mbh, &full[s], kr, 0);
        if (SPLIT) tma_load_2d(sBlo(s), mbl, &full[s], kr, 0);
        issued = kt + 1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_tf32(kBM, BN, /*a_mn=*/true, /*b_mn=*/false);
      for (int kt = 0; kt < nk; ++kt) {
        const int s = kt % S;
        const int r = DRAIN ? kt / RS::D : 0, j = DRAIN ? kt - r * RS::D : kt, bank = r & 1;
        if (DRAIN && j == 0 && r >= 2 && !waitp(&bfree[bank], ((r >> 1) - 1) & 1, limit, 7)) {
          *abort_flag = 1;
          break;
        }
        if (!waitp(SPLIT ? &conv[s] : &full[s], (kt / S) & 1, limit, 2) || *abort_flag) {
          *abort_flag = 1;
          break;
        }
        fence_after_sync();
        const uint32_t a = smem_u32(sA(s)), al = smem_u32(sAlo(s)), b = smem_u32(sB(s)), bl = smem_u32(sBlo(s));
        const int ai = DRAIN ? bank * RS::NPB + j % RS::NPB : kt % NACC;
        const int fresh = DRAIN ? RS::NPB : NACC;  // the first steps of a round (of the CTA) overwrite
        const uint32_t td = tmem + uint32_t(ai * kCols);
#pragma unroll
        for (int kk = 0; kk < kBK / 8; ++kk) {
          // A: 8 K-rows per MMA = two 512-byte atoms along K; B: 8 TF32 = 32 bytes along K
          const uint64_t da = sw128b32_mn_desc(a + kk * 1024, 4096, 512);
          const uint64_t db = sw128_kmajor(b + kk * 32);
          const uint32_t acc = (j >= fresh || kk > 0) ? 1u : 0u;
          mma_tf32(td, da, db, idesc, acc);
          if (SPLIT) {
            mma_tf32(td, da, sw128_kmajor(bl + kk * 32), idesc, 1u);
            mma_tf32(td, sw128b32_mn_desc(al + kk * 1024, 4096, 512), db, idesc, 1u);
          }
        }
        mma_commit(&empty[s]);
        if (DRAIN && (j == RS::D - 1 || kt == nk - 1)) mma_commit(&bfull[bank]);
      }
      mma_commit(accf);  // fires once every MMA issued above has completed
    }
  } else {
    // warps 2..5: split A (3xTF32), add finished rounds into registers, store
    // the partial tile; exit decisions are warp-uniform (TMEM loads are
    // warp-collective)
    const int t = threadIdx.x - 64;  // 0..127
    const int q = warp & 3;          // TMEM lane quadrant of this warp
    const uint32_t tlane = tmem + (uint32_t(q * 32) << 16);
    constexpr int NR = DRAIN ? BN : 16;
    float racc[NR];
#pragma unroll
    for (int i = 0; i < NR; ++i) racc[i] = 0.f;
    int drained = 0;
    auto drain = [&](int rr) -> bool {
      if (!__all_sync(0xffffffffu, waitp(&bfull[rr & 1], (rr >> 1) & 1, limit, 8))) return false;
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
        if (!__all_sync(0xffffffffu, waitp(&full[s], (kt / S) & 1, limit, 3) && !*abort_flag)) {
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
    bool ok = __all_sync(0xffffffffu, waitp(accf, 0, limit, 4) && !*abort_flag);
    fence_after_sync();
    if constexpr (DRAIN) {
      const int nrounds = (nk + RS::D - 1) / RS::D;
      while (ok && drained < nrounds) ok = drain(drained);
    }
    const int row = q * 32 + lane;
    float* dst = P.partial + size_t(blockIdx.x) * BN * kBM + row;
    const int nacc = nk < NACC ? nk : NACC;
#pragma unroll
    for (int c = 0; c < BN; c += 16) {
      float v[16];
      if (ok && nk > 0 && DRAIN) {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = racc[(c + i) % NR];
      } else if (ok && nk > 0) {
        tmem_ld16(tlane + uint32_t(c), v);
        for (int a = 1; a < nacc; ++a) {
          float w[16];
          tmem_ld16(tlane + uint32_t(a * kCols + c), w);
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] += w[i];
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) dst[size_t(c + i) * kBM] = v[i];  // [col][row]: coalesced over the warp
    }
  }
  // before exit: no copy and no MMA of this CTA may still be in flight
  if (warp == 0 && lane == 0 && *abort_flag) {
    for (int kt = (issued > S ? issued - S : 0); kt < issued; ++kt)
      waitp(&full[kt % S], (kt / S) & 1, kDrainLimitNs, 5);
  }
  if (warp == 1 && lane == 0) waitp(accf, 0, kDrainLimitNs, 6);
  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    tmem_dealloc(tmem, kAlloc);
  }
}

// ---- packing of x (and gg_x) for a chunk: Xt[u][K], K = s (2 l1 + 1) + m1 ----
struct XtBlock {
  int64_t off;  // float offset of the block inside one (pair, half) slice
  int in_off, c_in, n1, kpad;
};
struct XtParams {
  XtBlock b[kMaxBlocks];
  int n_in, dim_in, s0, nc;
  const float* x[2];
  float* hi[2];
  float* lo[2];
};

__global__ void k_pack_xt(const __grid_constant__ XtParams P) {
  const int pair = blockIdx.y / P.n_in, i1 = blockIdx.y - pair * P.n_in;
  const float* x = P.x[pair];
  if (!x) return;
  const XtBlock& B = P.b[i1];
  const int kreal = P.nc * B.n1;
  const int64_t n = int64_t(B.c_in) * B.kpad;
  float* hi = P.hi[pair] + B.off;
  float* lo = P.lo[pair] ? P.lo[pair] + B.off : nullptr;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const int u = int(i / B.kpad), K = int(i - int64_t(u) * B.kpad);
    float v = 0.f;
    if (K < kreal) {
      const int s = K / B.n1, m1 = K - s * B.n1;
      v = x[int64_t(P.s0 + s) * P.dim_in + B.in_off + u * B.n1 + m1];
    }
    if (lo) {
      const float h = rn_tf32(v);
      hi[i] = h;
      lo[i] = rn_tf32(v - h);
    } else {
      hi[i] = v;
    }
  }
}

// ---- ordered reduction of the partial tiles into dTheta ----
struct RedPath {
  int64_t theta_off;
  int c_in, c_out, g0, g1;  // groups of pair 0 / 1 (-1: none)
};
struct RedParams {
  RedPath p[kMaxPaths];
  DtGroup g[kMaxGroups];
  int R, BN;
  const float* partial;
};

__global__ void k_dtheta_reduce(const __grid_constant__ RedParams P, float* __restrict__ dtheta) {
  const RedPath& q = P.p[blockIdx.y];
  const int64_t n = int64_t(P.R) * q.c_in * q.c_out;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < n; e += int64_t(gridDim.x) * blockDim.x) {
    const int w = int(e % q.c_out);
    const int64_t t = e / q.c_out;
    const int u = int(t % q.c_in), k = int(t / q.c_in);
    const int i = k * q.c_out + w, mt = i >> 7, r = i & 127;
    float s = 0.f;
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      const int gi = pr == 0 ? q.g0 : q.g1;
      if (gi < 0) continue;
      const DtGroup& G = P.g[gi];
      const float* src = P.partial + (size_t(G.cta0 + mt * G.n_split) * P.BN + u) * kBM + r;
      for (int sp = 0; sp < G.n_split; ++sp) s += src[size_t(sp) * P.BN * kBM];
    }
    dtheta[q.theta_off + e] += s;
  }
}

// ---- host side ----------------------------------------------------------------
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

// fp32 [rows][cols] with row pitch ld floats; box box_cols x box_rows
bool make_map(CUtensorMap* m, const float* p, int64_t rows, int64_t cols, int64_t ld, int box_cols, int box_rows,
              CUtensorMapSwizzle swz) {
  EncodeFn enc = encoder();
  if (!enc) return false;
  if ((reinterpret_cast<uintptr_t>(p) & 15) || ((ld * 4) & 15) || rows <= 0 || cols <= 0) return false;
  cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(ld * 4)};
  cuuint32_t box[2] = {cuuint32_t(box_cols), cuuint32_t(box_rows)};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(p), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int64_t kpad_of(int nc, int n1) { return (int64_t(nc) * n1 + 3) & ~int64_t(3); }

template <int BN, bool SPLIT>
cudaError_t set_smem() {
  return cudaFuncSetAttribute(k_dtheta_tc<BN, SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              DtSmem<BN>::kBytes);
}

template <int BN, bool SPLIT>
cudaError_t launch(const DtParams& p, int n_cta, cudaStream_t st) {
  k_dtheta_tc<BN, SPLIT><<<n_cta, 192, DtSmem<BN>::kBytes, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

int dtheta_tc_bn(const DevPlan& d) {
  const int c = d.max_c_in;
  return c <= 32 ? 32 : c <= 64 ? 64 : c <= 128 ? 128 : 256;
}

bool dtheta_tc_shape_ok(const DevPlan& d) {
  if (d.family != TPCONV_FAMILY_FULL || d.P <= 0 || d.max_c_in > 256) return false;
  for (int i = 0; i < d.n_in; ++i)
    if (d.Kx[i] % 4) return false;
  for (int p = 0; p < d.P; ++p)
    if ((d.R * d.path[p].c_out) % 4 || d.path[p].kxoff % 4) return false;
  return true;
}

size_t dtheta_tc_xt_floats(const DevPlan& d, int64_t nc) {
  size_t n = 0;
  for (int i = 0; i < d.n_in; ++i) n += size_t(d.in_mul[i]) * kpad_of(int(nc), 2 * d.in_l[i] + 1);
  return 4 * ((n + 63) & ~size_t(63));  // 2 pairs x {hi, lo}
}

size_t dtheta_tc_partial_floats(const DevPlan& d) {
  // room for two waves of one CTA per SM, and for one K range per row tile of both pairs
  int64_t tiles = 0;
  for (int p = 0; p < d.P; ++p) tiles += 2 * ((d.R * d.path[p].c_out + kBM - 1) / kBM);
  return size_t(std::max<int64_t>(2 * kMaxSms, tiles)) * dtheta_tc_bn(d) * kBM;
}

cudaError_t dtheta_tc_init() {
  cudaError_t e = cudaSuccess;
  for (cudaError_t r : {set_smem<32, true>(), set_smem<64, true>(), set_smem<128, true>(), set_smem<256, true>(),
                        set_smem<32, false>(), set_smem<64, false>(), set_smem<128, false>(), set_smem<256, false>()})
    if (r != cudaSuccess && e == cudaSuccess) e = r;
  return e;
}

cudaError_t dtheta_tc_read_error(int* code) {
  int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(code, g_dt_error, sizeof(int));
  if (e) return e;
  return *code ? cudaMemcpyToSymbol(g_dt_error, &zero, sizeof(int)) : cudaSuccess;
}

cudaError_t dtheta_tc_accumulate(const DevPlan& d, int s0, int nc, const float* xa, const float* Ba,
                                 const float* xb, const float* Bb, float* dtheta, float* xt, float* partial,
                                 bool split, uint64_t wait_ns, cudaStream_t st) {
  const bool pa = xa && Ba, pb = xb && Bb;
  if (nc <= 0 || d.P <= 0 || (!pa && !pb)) return cudaSuccess;
  if (!dtheta_tc_shape_ok(d) || !encoder() || !xt || !partial) return cudaErrorInvalidValue;
  const int BN = dtheta_tc_bn(d);
  // ---- Xt of both pairs: [pair][half][blocks], one pack launch
  const size_t slice = dtheta_tc_xt_floats(d, nc) / 4;
  XtParams xp;
  std::memset(&xp, 0, sizeof(xp));
  xp.n_in = d.n_in;
  xp.dim_in = d.dim_in;
  xp.s0 = s0;
  xp.nc = nc;
  int64_t off = 0, nmax = 0;
  for (int i = 0; i < d.n_in; ++i) {
    const int n1 = 2 * d.in_l[i] + 1;
    xp.b[i] = XtBlock{off, d.in_off[i], d.in_mul[i], n1, int(kpad_of(nc, n1))};
    off += int64_t(d.in_mul[i]) * kpad_of(nc, n1);
    nmax = std::max<int64_t>(nmax, int64_t(d.in_mul[i]) * kpad_of(nc, n1));
  }
  const float* xs[2] = {pa ? xa : nullptr, pb ? xb : nullptr};
  for (int pr = 0; pr < 2; ++pr) {
    xp.x[pr] = xs[pr];
    xp.hi[pr] = xt + (2 * pr) * slice;
    xp.lo[pr] = split ? xt + (2 * pr + 1) * slice : nullptr;
  }
  {
    const int bx = int(std::min<int64_t>((nmax + 255) / 256, 4 * 148 / std::max(1, 2 * d.n_in) + 1));
    k_pack_xt<<<dim3(unsigned(bx), unsigned(2 * d.n_in)), 256, 0, st>>>(xp);
    cudaError_t e = cudaGetLastError();
    if (e) return e;
  }
  // ---- groups and their K ranges.  The range size kc (a multiple of 32) is
  // the one whose CTAs finish soonest: waves of one CTA per SM times the rows
  // of a range, over every kc whose CTAs fit the partial buffer.
  struct Gr {
    int pair, p, n_mt, K;
  };
  Gr gr[kMaxGroups];
  int ng = 0;
  for (int pr = 0; pr < 2; ++pr) {
    if (!(pr == 0 ? pa : pb)) continue;
    for (int p = 0; p < d.P; ++p) {
      const DevPath& q = d.path[p];
      gr[ng++] = Gr{pr, p, (d.R * q.c_out + kBM - 1) / kBM, nc * (2 * q.l1 + 1)};
    }
  }
  auto count = [&](int64_t kc) {
    int64_t n = 0;
    for (int i = 0; i < ng; ++i) n += int64_t(gr[i].n_mt) * ((gr[i].K + kc - 1) / kc);
    return n;
  };
  int64_t Kmax = 32;
  for (int i = 0; i < ng; ++i) Kmax = std::max<int64_t>(Kmax, gr[i].K);
  Kmax = (Kmax + 31) & ~int64_t(31);
  const int64_t cap = int64_t(dtheta_tc_partial_floats(d) / (size_t(BN) * kBM));
  const int64_t sms = sm_count() * dt_ctas_per_sm(BN);  // CTA slots of one wave
  int64_t best_kc = -1, best_cost = 0;
  for (int64_t kc = 32; kc <= Kmax; kc += 32) {
    const int64_t n = count(kc);
    if (n > cap) continue;
    const int64_t cost = ((n + sms - 1) / sms) * kc;
    if (best_kc < 0 || cost < best_cost) {
      best_kc = kc;
      best_cost = cost;
    }
  }
  if (best_kc < 0) return cudaErrorInvalidValue;  // the partial buffer is sized so that this cannot happen
  // ---- kernel parameters
  DtParams dp;
  RedParams rp;
  std::memset(&dp, 0, sizeof(dp));
  std::memset(&rp, 0, sizeof(rp));
  int mapped[2][kMaxBlocks];
  for (auto& r : mapped)
    for (int& v : r) v = -1;
  int nmap = 0, cta = 0;
  for (int i = 0; i < ng; ++i) {
    const DevPath& q = d.path[gr[i].p];
    const int i1 = q.i1, pr = gr[i].pair;
    if (mapped[pr][i1] < 0) {
      const int n1 = 2 * d.in_l[i1] + 1;
      const float* Bst = (pr == 0 ? Ba : Bb) + size_t(nc) * d.b_pref[i1];
      const float* xh = xp.hi[pr] + xp.b[i1].off;
      const float* xl = split ? xp.lo[pr] + xp.b[i1].off : xh;
      const int64_t K = int64_t(nc) * n1, kp = kpad_of(nc, n1);
      if (!make_map(&dp.a[nmap], Bst, K, d.Kx[i1], d.Kx[i1], 32, 32, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B) ||
          !make_map(&dp.bh[nmap], xh, d.in_mul[i1], K, kp, 32, BN, CU_TENSOR_MAP_SWIZZLE_128B) ||
          !make_map(&dp.bl[nmap], xl, d.in_mul[i1], K, kp, 32, BN, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
      mapped[pr][i1] = nmap++;
    }
    const int ns = int((gr[i].K + best_kc - 1) / best_kc);
    dp.g[i] = DtGroup{cta, gr[i].n_mt, ns, int(best_kc), gr[i].K, q.kxoff, mapped[pr][i1]};
    cta += gr[i].n_mt * ns;
  }
  dp.n_groups = ng;
  dp.partial = partial;
  dp.wait_ns = wait_ns;
  cudaError_t e;
  switch (BN) {
    case 32: e = split ? launch<32, true>(dp, cta, st) : launch<32, false>(dp, cta, st); break;
    case 64: e = split ? launch<64, true>(dp, cta, st) : launch<64, false>(dp, cta, st); break;
    case 128: e = split ? launch<128, true>(dp, cta, st) : launch<128, false>(dp, cta, st); break;
    default: e = split ? launch<256, true>(dp, cta, st) : launch<256, false>(dp, cta, st); break;
  }
  if (e) return e;
  rp.R = d.R;
  rp.BN = BN;
  rp.partial = partial;
  std::memcpy(rp.g, dp.g, sizeof(rp.g));
  int64_t emax = 0;
  for (int p = 0; p < d.P; ++p) {
    const DevPath& q = d.path[p];
    rp.p[p] = RedPath{q.theta_off, q.c_in, q.c_out, -1, -1};
    emax = std::max<int64_t>(emax, int64_t(d.R) * q.c_in * q.c_out);
  }
  for (int i = 0; i < ng; ++i) (gr[i].pair == 0 ? rp.p[gr[i].p].g0 : rp.p[gr[i].p].g1) = i;
  const int bx = int(std::min<int64_t>((emax + 255) / 256, std::max(1, 8 * 148 / d.P)));
  k_dtheta_reduce<<<dim3(unsigned(bx), unsigned(d.P)), 256, 0, st>>>(rp, dtheta);
  return cudaGetLastError();
}

}  // namespace tpc
