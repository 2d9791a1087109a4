// C ABI entry points of the streaming CG tensor-product convolution: argument
// checks, workspace carving, receiver / sender chunking and kernel launches.
//
// Schedule ("Sobek", arXiv 2607.18074, abstract): radial projection, spherical-
// harmonic coupling and aggregation are reassociated so that edge-local
// products land directly in bounded node-side state, which a node-level Theta
// contraction then mixes (fully connected C_in -> C_out per path).
//   forward : A = receiver stream, out = A . Theta               (per output block)
//   backward: G = g . Theta^T, receiver adjoint stream -> dY, db, dvec
//             B = sender stream over g, dx = B . Theta, dTheta = x^T B
// Node-side state is processed in chunks of receivers (senders) sized by the
// workspace cap, so its memory never depends on the edge count.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "gemm_simt.cuh"
#include "channelwise.h"
#include "dtheta.h"
#include "dtheta_tc.h"
#include "gemm_tc.h"
#include "graph.cuh"
#include "launchers.h"
#include "plan.h"
#include "wn_layout.h"
#include "workspace.h"

using namespace tpc;

namespace tpc {
std::vector<TuInit>& tu_registry() {
  static std::vector<TuInit> r;
  return r;
}
}  // namespace tpc

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned long long g_ready_ctx[kMaxDevices];  // id of the context set up per device (0 = none)

// Id of the current CUDA context (driver entry point, looked up once); 0 when
// unavailable.  A device reset destroys the context and with it the constant
// tables, so the set-up below is keyed on the context, not on the device.
unsigned long long current_context_id() {
  using GetCur = int (*)(void**);
  using GetId = int (*)(void*, unsigned long long*);
  static GetCur get_cur = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<GetCur>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
  });
  void* ctx = nullptr;
  unsigned long long id = 0;
  if (!get_cur || !get_id || get_cur(&ctx) != 0 || !ctx || get_id(ctx, &id) != 0) return 0;
  return id;
}

// Once per device context: upload the real-CG table and raise the kernels'
// shared memory limit.  The first call in a context synchronises the device
// (cudaMemcpyToSymbol), so it must not happen inside a stream capture.
int ensure_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TPCONV_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  const unsigned long long ctx = current_context_id();
  if (g_ready_ctx[dev] != 0 && (ctx == 0 || g_ready_ctx[dev] == ctx)) return TPCONV_OK;
  const float* t = cg_table_f32();
  if (!t) return TPCONV_ERR_INTERNAL;
  for (const TuInit& tu : tu_registry()) {
    if (tu.upload(t) != cudaSuccess) return TPCONV_ERR_CUDA;
    if (tu.smem && tu.smem(227 * 1024) != cudaSuccess) return TPCONV_ERR_CUDA;
  }
  if (dtheta_smem_init() != cudaSuccess) return TPCONV_ERR_CUDA;
  if (gemm_tc_init() != cudaSuccess) return TPCONV_ERR_CUDA;
  if (dtheta_tc_init() != cudaSuccess) return TPCONV_ERR_CUDA;
  const unsigned long long now = current_context_id();  // the set-up above created the context if needed
  g_ready_ctx[dev] = now ? now : ~0ull;
  return TPCONV_OK;
}

// Limit of every wait of the tensor-core kernels on their own pipelines (set by
// tpconv_set_wait_limit; read when a call is issued).
std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};
inline uint64_t wait_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

// 16-byte aligned (or null): the adjoint streams stage feature rows with 16-byte copies
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// ---- diagnostics: per-phase launch counts and optional event timing ----
struct Profiler {
  std::mutex mu;
  bool on = false;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pending[TPCONV_N_PHASES];
  double ms[TPCONV_N_PHASES] = {};
  std::atomic<int64_t> launches[TPCONV_N_PHASES];
  Profiler() {
    for (auto& l : launches) l = 0;
  }
};
Profiler& prof() {
  static Profiler p;
  return p;
}
inline void note(int phase, int64_t n) { prof().launches[phase] += n; }

// Brackets one phase of a call with events on the call's stream (when enabled).
struct PhaseScope {
  int phase;
  cudaStream_t st;
  cudaEvent_t a = nullptr, b = nullptr;
  PhaseScope(int ph, cudaStream_t s) : phase(ph), st(s) {
    Profiler& p = prof();
    if (!p.on) return;
    if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) return;
    cudaEventRecord(a, st);
  }
  ~PhaseScope() {
    if (!b) return;
    cudaEventRecord(b, st);
    Profiler& p = prof();
    std::lock_guard<std::mutex> lk(p.mu);
    p.pending[phase].push_back({a, b});
  }
};

inline cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline float* F(const float* p) { return const_cast<float*>(p); }

int first_path_of_out_block(const DevPlan& d, int i3) {
  for (int p = 0; p < d.P; ++p)
    if (d.path[p].i3 == i3) return p;
  return -1;
}

int check_ws(const tpconv_plan* plan, int op, int64_t N, int64_t E, void* ws, size_t ws_bytes, WsLayout* L) {
  int st = ws_layout(*plan, op, N, E, L);
  if (st) return st;
  if (ws_bytes < L->total) return TPCONV_ERR_WORKSPACE_TOO_SMALL;
  if (L->total > 0 && (!ws || (reinterpret_cast<uintptr_t>(ws) & 255))) return TPCONV_ERR_INVALID_ARG;
  return TPCONV_OK;
}

// Theta^T of every output block (tensor-core B operand): hi (and lo for 3xTF32)
// at the block's Theta offset inside the workspace's Theta region.
cudaError_t prep_theta_T(const tpconv_plan* plan, const float* theta, float* hi, float* lo, cudaStream_t st) {
  const DevPlan& d = plan->dp;
  for (int i3 = 0; i3 < d.n_out; ++i3) {
    const int p0 = first_path_of_out_block(d, i3);
    if (p0 < 0) continue;
    const int64_t off = d.path[p0].theta_off;
    cudaError_t e = split_transpose(theta + off, d.Kb[i3], d.out_mul[i3], hi + off, lo ? lo + off : nullptr, st);
    if (e) return e;
  }
  return cudaSuccess;
}

bool use_tc(const tpconv_plan* plan) {
  return plan->dp.family == TPCONV_FAMILY_FULL &&
         (plan->opt.gemm == TPCONV_GEMM_FP32 || plan->opt.gemm == TPCONV_GEMM_TF32);
}
bool channelwise(const tpconv_plan* plan) { return plan->dp.family == TPCONV_FAMILY_CHANNELWISE; }

// out[r0 : r0+nc] = A . Theta (mode 0) or += (mode 1), per output block.  With
// thT (Theta^T hi, lo) the tensor-core GEMM runs, else the FFMA GEMM.
// ---- fork / join of independent launches ----------------------------------
// The per-block Theta contractions of one call are independent (disjoint
// output blocks) but each launch alone fills the GPU unevenly (e.g. 32, 96 and
// 160 tiles of one CTA per SM); issuing them on side streams lets their waves
// overlap.  Side streams and events are created once per host thread and
// device; the fork is an event on the caller's stream that each side stream
// waits for, the join an event per side stream the caller's stream waits for,
// so the call stays ordered on the caller's stream (and capturable as a fork /
// join graph once the side resources exist).
constexpr int kSide = 2;
struct SideRes {
  cudaStream_t s[kSide] = {};
  cudaEvent_t fork = nullptr, join[kSide] = {};
  bool ok = false;
};
SideRes* side_res() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  thread_local SideRes r[kMaxDevices];
  SideRes& x = r[dev];
  if (!x.ok) {
    bool ok = cudaEventCreateWithFlags(&x.fork, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; i < kSide && ok; ++i)
      ok = cudaStreamCreateWithFlags(&x.s[i], cudaStreamNonBlocking) == cudaSuccess &&
           cudaEventCreateWithFlags(&x.join[i], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) return nullptr;  // fall back to the caller's stream
    x.ok = true;
  }
  return &x;
}
class ForkJoin {
 public:
  explicit ForkJoin(cudaStream_t main) : main_(main), r_(side_res()) {}
  // stream for the i-th independent piece of work
  cudaStream_t stream(int i) {
    const int k = i % (kSide + 1);
    if (k == 0 || !r_) return main_;
    if (!forked_) {
      if (cudaEventRecord(r_->fork, main_) != cudaSuccess) return main_;
      forked_ = true;
    }
    if (!used_[k - 1]) {
      if (cudaStreamWaitEvent(r_->s[k - 1], r_->fork, 0) != cudaSuccess) return main_;
      used_[k - 1] = true;
    }
    return r_->s[k - 1];
  }
  cudaError_t join() {
    for (int k = 0; k < kSide; ++k) {
      if (!used_[k]) continue;
      cudaError_t e = cudaEventRecord(r_->join[k], r_->s[k]);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(main_, r_->join[k], 0);
      if (e != cudaSuccess) return e;
      used_[k] = false;
    }
    return cudaSuccess;
  }
  ~ForkJoin() { join(); }

 private:
  cudaStream_t main_;
  SideRes* r_;
  bool forked_ = false;
  bool used_[kSide] = {};
};

cudaError_t node_mix_forward(const tpconv_plan* plan, int r0, int nc, const float* A, const float* theta,
                             const float* thT_hi, const float* thT_lo, float* out, cudaStream_t st, int mode = 0) {
  const DevPlan& d = plan->dp;
  if (channelwise(plan)) return cw_forward(d, r0, nc, A, theta, out, mode, st);
  ForkJoin fj(st);
  for (int i3 = 0; i3 < d.n_out; ++i3) {
    cudaStream_t si = fj.stream(i3);
    const int n3 = 2 * d.out_l[i3] + 1, cout = d.out_mul[i3];
    const int p0 = first_path_of_out_block(d, i3);
    const int64_t toff = p0 >= 0 ? d.path[p0].theta_off : 0;
    const float* Ab = A + size_t(nc) * d.a_pref[i3];
    const int Kb = d.Kb[i3];
    const int64_t M = int64_t(nc) * n3;
    if (thT_hi && Kb > 0 && gemm_tc_supported(Ab, Kb, thT_hi + toff, Kb, int(M), cout, Kb)) {
      TcOut o{out + size_t(r0) * d.dim_out + d.out_off[i3], n3, d.dim_out, 1, n3};
      const bool split = plan->opt.gemm == TPCONV_GEMM_FP32;
      cudaError_t e = gemm_tc(Ab, Kb, thT_hi + toff, split ? thT_lo + toff : nullptr, Kb, int(M), cout, Kb, o,
                              mode, split, si, wait_ns());
      if (e) return e;
      continue;
    }
    MView a = mrow(F(Ab), Kb);
    MView b = mrow(F(theta + toff), cout);
    MView c = mview(out + size_t(r0) * d.dim_out + d.out_off[i3], n3, d.dim_out, 1, 1, n3, 0);
    cudaError_t e = gemm_simt(M, cout, Kb, a, b, c, mode, si);
    if (e) return e;
  }
  return fj.join();
}

// Theta operands of the tensor-core contractions for one Theta (slot 0: Theta,
// slot 1: gg_Theta), carved from the workspace's Theta region:
//   T  = per output block Theta_blk^T [C_out][K_b]   (out / d_g = A . Theta)
//   N  = Theta itself, split elementwise              (G = g . Theta^T)
//   X  = per input block [C_in][K_x]                  (dx = B . Theta)
// hi / lo are the 3xTF32 halves; lo is null in TF32 mode.
struct TcTheta {
  const float *T_hi = nullptr, *T_lo = nullptr, *N_hi = nullptr, *N_lo = nullptr, *X_hi = nullptr, *X_lo = nullptr;
};

int64_t x_block_off(const DevPlan& d, int i1) {
  int64_t o = 0;
  for (int i = 0; i < i1; ++i) o += int64_t(d.in_mul[i]) * d.Kx[i];
  return o;
}

// kernel launches of prep_tc_theta
int64_t tc_theta_launches(const DevPlan& d, bool needT, bool needN, bool needX) {
  int64_t n = (needN ? 1 : 0) + (needX && d.P > 0 ? 1 : 0);
  if (needT)
    for (int i3 = 0; i3 < d.n_out; ++i3) n += first_path_of_out_block(d, i3) >= 0;
  return n;
}

cudaError_t prep_tc_theta(const tpconv_plan* plan, int op, const float* theta, float* region, int slot, bool needT,
                          bool needN, bool needX, TcTheta* o, cudaStream_t st) {
  const DevPlan& d = plan->dp;
  const size_t tn = (plan->theta_numel + 63) & ~size_t(63);
  const bool split = plan->opt.gemm == TPCONV_GEMM_FP32;
  // slice (kind, half) of this slot; null when the operation reserves none
  auto sl = [&](int kind, int half) -> float* {
    const int i = theta_region(op, slot, kind, half, true, split);
    return i < 0 ? nullptr : region + size_t(i) * tn;
  };
  cudaError_t e;
  if (needT) {
    float *hi = sl(kThetaT, 0), *lo = sl(kThetaT, 1);
    if (!hi || (split && !lo)) return cudaErrorInvalidValue;
    if ((e = prep_theta_T(plan, theta, hi, lo, st))) return e;
    o->T_hi = hi;
    o->T_lo = lo;
  }
  if (needN) {
    float *hi = sl(kThetaN, 0), *lo = sl(kThetaN, 1);
    if (!hi || (split && !lo)) return cudaErrorInvalidValue;
    if ((e = split_elementwise(theta, int64_t(plan->theta_numel), hi, lo, st))) return e;
    o->N_hi = hi;
    o->N_lo = lo;
  }
  if (needX) {
    float *hi = sl(kThetaX, 0), *lo = sl(kThetaX, 1);
    if (!hi || (split && !lo)) return cudaErrorInvalidValue;
    static_assert(kXPackMax >= kMaxPaths, "one launch packs every path");
    XPackList xl;
    xl.n = d.P;
    xl.R = d.R;
    for (int p = 0; p < d.P; ++p) {
      const DevPath& q = d.path[p];
      xl.p[p] = XPackPath{q.theta_off, x_block_off(d, q.i1), q.c_in, q.c_out, q.kxoff, d.Kx[q.i1]};
    }
    if ((e = theta_x_pack_all(theta, xl, hi, lo, st))) return e;
    o->X_hi = hi;
    o->X_lo = lo;
  }
  return cudaSuccess;
}

// G[r0 : r0+nc] = g . Theta^T  (per output block); gpack: nc * dim_out floats of scratch
cudaError_t node_mix_adjoint(const tpconv_plan* plan, int r0, int nc, const float* g, const float* theta,
                             const TcTheta* tc, float* gpack, float* G, cudaStream_t st) {
  const DevPlan& d = plan->dp;
  if (channelwise(plan)) return cw_adjoint(d, r0, nc, g, theta, G, st);
  ForkJoin fj(st);
  for (int i3 = 0; i3 < d.n_out; ++i3) {
    if (d.Kb[i3] == 0) continue;
    cudaStream_t si = fj.stream(i3);
    float* gp = gpack + size_t(nc) * d.out_off[i3];  // this block's slice of the pack region
    const int n3 = 2 * d.out_l[i3] + 1, cout = d.out_mul[i3];
    const int p0 = first_path_of_out_block(d, i3);
    const int64_t toff = d.path[p0].theta_off;
    float* Gb = G + size_t(nc) * d.a_pref[i3];
    const int64_t M = int64_t(nc) * n3;
    cudaError_t e;
    if (tc && tc->N_hi && gemm_tc_supported(gp, cout, tc->N_hi + toff, cout, int(M), d.Kb[i3], cout) &&
        (d.Kb[i3] & 3) == 0) {
      if ((e = pack_rows(g, d.dim_out, d.out_off[i3], cout, n3, r0, nc, gp, si))) return e;
      TcOut o{Gb, 1, d.Kb[i3], 0, 1};
      const bool split = tc->N_lo != nullptr;
      if ((e = gemm_tc(gp, cout, tc->N_hi + toff, split ? tc->N_lo + toff : nullptr, cout, int(M), d.Kb[i3], cout,
                       o, 0, split, si, wait_ns())))
        return e;
      continue;
    }
    MView a = mview(F(g) + size_t(r0) * d.dim_out + d.out_off[i3], n3, d.dim_out, 1, 1, n3, 0);
    MView b = mview(F(theta) + toff, 1, 1, 0, 1, cout, 0);
    MView c = mrow(Gb, d.Kb[i3]);
    if ((e = gemm_simt(M, d.Kb[i3], cout, a, b, c, 0, si))) return e;
  }
  return fj.join();
}

// dtheta += xa^T Ba (+ xb^T Bb) over the senders s0 : s0+nc: on the tensor
// cores (deterministic split-K) where the workspace holds their regions, else
// the FFMA kernel.
cudaError_t theta_gradient(const tpconv_plan* plan, const WsLayout& L, void* ws, int s0, int nc, const float* xa,
                           const float* Ba, const float* xb, const float* Bb, float* dtheta, cudaStream_t st) {
  const DevPlan& d = plan->dp;
  if (use_tc(plan) && L.xt_bytes > 0 && L.part_bytes > 0) {
    char* w = static_cast<char*>(ws);
    return dtheta_tc_accumulate(d, s0, nc, xa, Ba, xb, Bb, dtheta, reinterpret_cast<float*>(w + L.off_xt),
                                reinterpret_cast<float*>(w + L.off_part), plan->opt.gemm == TPCONV_GEMM_FP32,
                                wait_ns(), st);
  }
  return dtheta_accumulate(d, s0, nc, xa, Ba, xb, Bb, dtheta, st);
}

// kernel launches of theta_gradient: pack, GEMM and ordered reduce, or one FFMA kernel
int64_t theta_gradient_launches(const tpconv_plan* plan, const WsLayout& L) {
  return (use_tc(plan) && L.xt_bytes > 0 && L.part_bytes > 0) ? 3 : 1;
}

// dx[s0 : s0+nc] += B . Theta (per input block) and dtheta += x^T B (per path)
cudaError_t node_mix_sender(const tpconv_plan* plan, const WsLayout& L, void* ws, int s0, int nc, const float* B,
                            const float* x, const float* theta, const TcTheta* tc, float* dx, float* dtheta,
                            cudaStream_t st) {
  const DevPlan& d = plan->dp;
  cudaError_t e;
  if (channelwise(plan)) {
    if (dx && (e = cw_dx(d, s0, nc, B, theta, dx, st))) return e;
    return dtheta ? cw_dtheta(d, s0, nc, x, B, nullptr, nullptr, dtheta, st) : cudaSuccess;
  }
  ForkJoin fj(st);
  if (dx) {
    for (int i1 = 0; i1 < d.n_in; ++i1) {
      const int Kx = d.Kx[i1];
      if (Kx == 0) continue;
      cudaStream_t si = fj.stream(i1 + 1);  // the Theta gradient runs on the caller's stream
      const int n1 = 2 * d.in_l[i1] + 1, cin = d.in_mul[i1];
      const float* Bb = B + size_t(nc) * d.b_pref[i1];
      const int64_t M = int64_t(nc) * n1;
      if (tc && tc->X_hi) {
        const int64_t xo = x_block_off(d, i1);
        if (gemm_tc_supported(Bb, Kx, tc->X_hi + xo, Kx, int(M), cin, Kx)) {
          TcOut o{dx + size_t(s0) * d.dim_in + d.in_off[i1], n1, d.dim_in, 1, n1};
          const bool split = tc->X_lo != nullptr;
          if ((e = gemm_tc(Bb, Kx, tc->X_hi + xo, split ? tc->X_lo + xo : nullptr, Kx, int(M), cin, Kx, o, 1, split,
                           si, wait_ns())))
            return e;
          continue;
        }
      }
      for (int p = 0; p < d.P; ++p) {
        const DevPath& q = d.path[p];
        if (q.i1 != i1) continue;
        MView bp = mrow(F(B) + size_t(nc) * d.b_pref[q.i1] + q.kxoff, Kx);
        MView th = mview(F(theta) + q.theta_off, q.c_out, int64_t(q.c_in) * q.c_out, 1, 1, q.c_out, 0);
        MView c = mview(dx + size_t(s0) * d.dim_in + q.in_off, n1, d.dim_in, 1, 1, n1, 0);
        if ((e = gemm_simt(M, q.c_in, int64_t(d.R) * q.c_out, bp, th, c, 1, si))) return e;
      }
    }
  }
  if (dtheta && (e = theta_gradient(plan, L, ws, s0, nc, x, B, nullptr, nullptr, dtheta, st))) return e;
  return fj.join();
}

// ---- work lists of the edge streams (graph.cuh) ------------------------------
struct WorkList {
  int* counter;
  int* extra;  // exclusive scan of the nodes' extra items; extra[nc] = their total
};
WorkList work_list(const WsLayout& L, void* ws, int which, int64_t chunk_nodes) {
  int* base = reinterpret_cast<int*>(static_cast<char*>(ws) + L.off_lists) + size_t(which) * L.list_ints;
  return WorkList{base, base + 32 + work_list_pad(chunk_nodes)};
}
// pieces of at most seg edges for the nodes n0 .. n0+nc-1 of ptr; resets the counter
cudaError_t build_work_list(const WorkList& wl, const WsLayout& L, const int* ptr, int n0, int nc, int seg,
                            cudaStream_t s) {
  (void)L;
  k_build_work_list<<<1, 1024, 0, s>>>(nc, ptr, n0, seg, wl.extra, wl.counter);
  return cudaGetLastError();
}
// piece length of the channel-lane streams: nodes far above the mean degree split
int piece_edges(int64_t N, int64_t E) {
  const int64_t mean = N > 0 ? (E + N - 1) / N : 0;
  return int(std::max<int64_t>(256, 4 * mean));
}
// ---- validate mode: the graph is checked on the device before any stream runs ----
__device__ int g_graph_error;

// rowptr non-decreasing from 0 to E, senders in [0, N), edge vectors finite and nonzero
__global__ void k_validate_graph(int64_t N, int64_t E, const int32_t* __restrict__ rowptr,
                                 const int32_t* __restrict__ col, const float* __restrict__ vec) {
  int bad = 0;
  const int64_t n = N + 1 > E ? N + 1 : E;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    if (i < N && rowptr[i] > rowptr[i + 1]) bad = 1;
    if (i == 0 && (rowptr[0] != 0 || int64_t(rowptr[N]) != E)) bad = 1;
    if (i < E) {
      const int32_t c = col[i];
      if (c < 0 || int64_t(c) >= N) bad = 1;
      if (vec) {
        const float x = vec[3 * i], y = vec[3 * i + 1], z = vec[3 * i + 2];
        const float r2 = x * x + y * y + z * z;
        if (!(r2 > 0.f) || !isfinite(r2)) bad = 1;
      }
    }
  }
  if (bad) atomicOr(&g_graph_error, 1);
}

// With plan->opt.validate set: check the receiver CSR (and edge vectors) and
// wait for the answer; TPCONV_ERR_GRAPH_INVALID stops the call before any
// kernel reads the graph.  Otherwise a no-op.
int validate_graph(const tpconv_plan* plan, int64_t N, int64_t E, const int32_t* rowptr, const int32_t* col,
                   const float* vec, cudaStream_t s) {
  if (!plan->opt.validate) return TPCONV_OK;
  const int zero = 0;
  int flag = 0;
  if (cudaMemcpyToSymbolAsync(g_graph_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s)) return TPCONV_ERR_CUDA;
  const int64_t n = std::max<int64_t>(N + 1, E);
  const unsigned blocks = unsigned(std::min<int64_t>((n + 255) / 256, 148 * 8));
  k_validate_graph<<<blocks, 256, 0, s>>>(N, E, rowptr, col, vec);
  if (cudaGetLastError()) return TPCONV_ERR_CUDA;
  if (cudaMemcpyFromSymbolAsync(&flag, g_graph_error, sizeof(int), 0, cudaMemcpyDeviceToHost, s)) return TPCONV_ERR_CUDA;
  if (cudaStreamSynchronize(s)) return TPCONV_ERR_CUDA;
  return flag ? TPCONV_ERR_GRAPH_INVALID : TPCONV_OK;
}

int finish(cudaError_t e) {
  if (e != cudaSuccess) return TPCONV_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? TPCONV_OK : TPCONV_ERR_CUDA;
}

// Synchronises s, then reads and clears the error records of the tensor-core
// kernels: TPCONV_ERR_TIMEOUT if a wait expired since the last read.
int device_status(cudaStream_t s, int* status) {
  *status = TPCONV_OK;
  if (cudaStreamSynchronize(s) != cudaSuccess) return TPCONV_ERR_CUDA;
  int a = 0, b = 0;
  if (gemm_tc_read_error(&a) != cudaSuccess || dtheta_tc_read_error(&b) != cudaSuccess) return TPCONV_ERR_CUDA;
  if (a || b) *status = TPCONV_ERR_TIMEOUT;
  return TPCONV_OK;
}

// end of a call: in validate mode the call waits for its kernels and reports an
// expired device wait as TPCONV_ERR_TIMEOUT
int finish_call(const tpconv_plan* plan, cudaStream_t s, cudaError_t e) {
  const int st = finish(e);
  if (st != TPCONV_OK || !plan->opt.validate) return st;
  int dst = TPCONV_OK;
  if (device_status(s, &dst) != TPCONV_OK) return TPCONV_ERR_CUDA;
  return dst;
}

}  // namespace

extern "C" {

int tpconv_get_device_status(const tpconv_plan* plan, void* stream, int* status) {
  if (!plan || !status) return TPCONV_ERR_INVALID_ARG;
  return device_status(S(stream), status);
}

int tpconv_set_wait_limit(uint64_t ns) {
  g_wait_ns.store(ns ? ns : kDefaultWaitNs, std::memory_order_relaxed);
  return TPCONV_OK;
}

int tpconv_profile_enable(int on) {
  prof().on = on != 0;
  return TPCONV_OK;
}

int tpconv_profile_reset(void) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> lk(p.mu);
  for (int i = 0; i < TPCONV_N_PHASES; ++i) {
    for (auto& ev : p.pending[i]) {
      cudaEventSynchronize(ev.second);
      cudaEventDestroy(ev.first);
      cudaEventDestroy(ev.second);
    }
    p.pending[i].clear();
    p.ms[i] = 0.0;
    p.launches[i] = 0;
  }
  return TPCONV_OK;
}

int tpconv_profile_read(int phase, double* ms, int64_t* launches) {
  if (phase < 0 || phase >= TPCONV_N_PHASES) return TPCONV_ERR_INVALID_ARG;
  Profiler& p = prof();
  std::lock_guard<std::mutex> lk(p.mu);
  for (auto& ev : p.pending[phase]) {
    float t = 0.f;
    if (cudaEventSynchronize(ev.second) != cudaSuccess) return TPCONV_ERR_CUDA;
    if (cudaEventElapsedTime(&t, ev.first, ev.second) != cudaSuccess) return TPCONV_ERR_CUDA;
    p.ms[phase] += t;
    cudaEventDestroy(ev.first);
    cudaEventDestroy(ev.second);
  }
  p.pending[phase].clear();
  if (ms) *ms = p.ms[phase];
  if (launches) *launches = p.launches[phase];
  return TPCONV_OK;
}

int tpconv_graph_transpose(const tpconv_plan* plan, int64_t N, int64_t E, const int32_t* rowptr,
                           const int32_t* col, int32_t* perm, int32_t* s_rowptr, int32_t* s_recv,
                           void* workspace, size_t workspace_bytes, void* stream) {
  if (!plan || N < 0 || E < 0) return TPCONV_ERR_INVALID_ARG;
  if (!s_rowptr || !rowptr || (E > 0 && (!col || !perm || !s_recv))) return TPCONV_ERR_INVALID_ARG;
  WsLayout L;
  int st = check_ws(plan, TPCONV_OP_TRANSPOSE, N, E, workspace, workspace_bytes, &L);
  if (st) return st;
  cudaStream_t s = S(stream);
  if ((st = ensure_device())) return st;
  if ((st = validate_graph(plan, N, E, rowptr, col, nullptr, s))) return st;
  PhaseScope ps(TPCONV_PHASE_TRANSPOSE, s);
  char* ws = static_cast<char*>(workspace);
  int* cnt = reinterpret_cast<int*>(ws + L.off_cursor);
  int* bsum = reinterpret_cast<int*>(ws + L.off_scan);
  int* tmp = reinterpret_cast<int*>(ws + L.off_tmp);
  if (cudaMemsetAsync(cnt, 0, size_t(N + 1) * 4, s)) return TPCONV_ERR_CUDA;
  if (E > 0) {
    k_count_senders<<<1184, 256, 0, s>>>(E, col, cnt);
    note(TPCONV_PHASE_TRANSPOSE, 1);
  }
  const int64_t n = N + 1;  // scan N+1 counts (last is 0) so s_rowptr[N] = E
  const int nb = int((n + 1023) / 1024);
  k_scan_blocks<<<nb, 1024, 0, s>>>(n, cnt, s_rowptr, bsum);
  k_scan_totals<<<1, 1024, 0, s>>>(nb, bsum, bsum + nb);
  k_scan_add<<<nb, 1024, 0, s>>>(n, s_rowptr, bsum);
  note(TPCONV_PHASE_TRANSPOSE, 3);
  if (E > 0) {
    if (cudaMemsetAsync(cnt, 0, size_t(N + 1) * 4, s)) return TPCONV_ERR_CUDA;
    k_fill_senders<<<1184, 128, 0, s>>>(N, rowptr, col, s_rowptr, cnt, tmp);
    k_sort_segments<<<2368, 256, 0, s>>>(N, rowptr, s_rowptr, tmp, perm, s_recv);
    note(TPCONV_PHASE_TRANSPOSE, 2);
  }
  return finish(cudaSuccess);
}

int tpconv_forward(const tpconv_plan* plan, int64_t N, int64_t E, const int32_t* rowptr, const int32_t* col,
                   const float* edge_vec, const float* x, const float* theta, float* out, void* workspace,
                   size_t workspace_bytes, void* stream) {
  if (!plan || N < 0 || E < 0) return TPCONV_ERR_INVALID_ARG;
  if (N > 0 && (!rowptr || !x || !out || !theta)) return TPCONV_ERR_INVALID_ARG;
  if (E > 0 && (!col || !edge_vec)) return TPCONV_ERR_INVALID_ARG;
  WsLayout L;
  int st = check_ws(plan, TPCONV_OP_FORWARD, N, E, workspace, workspace_bytes, &L);
  if (st) return st;
  if ((st = ensure_device())) return st;
  if (N == 0) return TPCONV_OK;
  const DevPlan& d = plan->dp;
  cudaStream_t s = S(stream);
  if ((st = validate_graph(plan, N, E, rowptr, col, edge_vec, s))) return st;
  float* A = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.off_state);
  float* treg = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.off_theta);
  const float* thT_hi = nullptr;
  const float* thT_lo = nullptr;
  if (use_tc(plan)) {
    PhaseScope ps(TPCONV_PHASE_OTHER, s);
    TcTheta tc;
    if (prep_tc_theta(plan, TPCONV_OP_FORWARD, theta, treg, 0, true, false, false, &tc, s)) return TPCONV_ERR_CUDA;
    thT_hi = tc.T_hi;
    thT_lo = tc.T_lo;
    note(TPCONV_PHASE_OTHER, tc_theta_launches(d, true, false, false));
  }
  for (int64_t r0 = 0; r0 < N; r0 += L.chunk_nodes) {
    const int nc = int(std::min<int64_t>(L.chunk_nodes, N - r0));
    {
      PhaseScope ps(TPCONV_PHASE_FWD_EDGE, s);
      const WorkList wl = work_list(L, workspace, 0, L.chunk_nodes);
      const int seg = piece_edges(N, E);
      if (build_work_list(wl, L, rowptr, int(r0), nc, seg, s)) return TPCONV_ERR_CUDA;
      if (TPC_WN_CALL_CPL(d, launch_wn_fwd, d, int(r0), nc, rowptr, col, edge_vec, x, A, wl.extra, wl.counter, seg,
                          s))
        return TPCONV_ERR_CUDA;
      note(TPCONV_PHASE_FWD_EDGE, 3);  // list, two stream launches
    }
    {
      PhaseScope ps(TPCONV_PHASE_FWD_NODE, s);
      if (node_mix_forward(plan, int(r0), nc, A, theta, thT_hi, thT_lo, out, s)) return TPCONV_ERR_CUDA;
      note(TPCONV_PHASE_FWD_NODE, d.n_out);
    }
  }
  return finish_call(plan, s, cudaSuccess);
}

int tpconv_backward(const tpconv_plan* plan, int64_t N, int64_t E, const int32_t* rowptr, const int32_t* col,
                    const int32_t* perm, const int32_t* s_rowptr, const int32_t* s_recv, const float* edge_vec,
                    const float* x, const float* theta, const float* g, float* dx, float* dtheta, float* dvec,
                    float* dY, float* db, void* workspace, size_t workspace_bytes, void* stream) {
  if (!plan || N < 0 || E < 0) return TPCONV_ERR_INVALID_ARG;
  const bool want_edge = dvec || dY || db;
  const bool want_node = dx || dtheta;
  if (N > 0 && (!rowptr || !x || !theta || !g)) return TPCONV_ERR_INVALID_ARG;
  if (E > 0 && (!col || !edge_vec)) return TPCONV_ERR_INVALID_ARG;
  if (want_node && N > 0 && (!s_rowptr || (E > 0 && (!perm || !s_recv)))) return TPCONV_ERR_INVALID_ARG;
  WsLayout L;
  int st = check_ws(plan, TPCONV_OP_BACKWARD, N, E, workspace, workspace_bytes, &L);
  if (st) return st;
  if ((st = ensure_device())) return st;
  const DevPlan& d = plan->dp;
  cudaStream_t s = S(stream);
  if (N > 0 && (st = validate_graph(plan, N, E, rowptr, col, edge_vec, s))) return st;
  if (dtheta && cudaMemsetAsync(dtheta, 0, plan->theta_numel * 4, s)) return TPCONV_ERR_CUDA;
  if (dx && N > 0 && cudaMemsetAsync(dx, 0, size_t(N) * d.dim_in * 4, s)) return TPCONV_ERR_CUDA;
  if (N == 0) return finish(cudaSuccess);
  float* S_ = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.off_state);
  float* treg = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.off_theta);
  float* gpack = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.off_pack);
  TcTheta tc;
  const TcTheta* tcp = nullptr;
  if (use_tc(plan)) {
    PhaseScope ps(TPCONV_PHASE_OTHER, s);
    if (prep_tc_theta(plan, TPCONV_OP_BACKWARD, theta, treg, 0, false, want_edge && E > 0, dx != nullptr, &tc, s)) return TPCONV_ERR_CUDA;
    note(TPCONV_PHASE_OTHER, tc_theta_launches(d, false, want_edge && E > 0, dx != nullptr));
    tcp = &tc;
  }
  if (want_edge && E > 0) {
    for (int64_t r0 = 0; r0 < N; r0 += L.chunk_nodes) {
      const int nc = int(std::min<int64_t>(L.chunk_nodes, N - r0));
      {
        PhaseScope ps(TPCONV_PHASE_BWD_NODE_G, s);
        if (node_mix_adjoint(plan, int(r0), nc, g, theta, tcp, gpack, S_, s)) return TPCONV_ERR_CUDA;
        note(TPCONV_PHASE_BWD_NODE_G, channelwise(plan) ? cw_launches_out(d) : 2 * d.n_out);
      }
      {
        PhaseScope ps(TPCONV_PHASE_BWD_EDGE_R, s);
        const bool wn = d.wn_ok && aligned16(x);
        const WorkList wl = work_list(L, workspace, 1, L.chunk_nodes);
        if (wn && build_work_list(wl, L, rowptr, int(r0), nc, kBatchEdges, s)) return TPCONV_ERR_CUDA;
        cudaError_t e = wn
                            ? TPC_WN_CALL(d, launch_wn_adj, d, int(r0), nc, rowptr, col, edge_vec, x, S_, dvec, dY, db,
                                          wl.extra, wl.counter, s)
                            : TPC_RM_CALL(d.rm, launch_radj_rm, d, int(r0), nc, rowptr, col, edge_vec, x, S_, dvec,
                                          dY, db, s);
        if (e) return TPCONV_ERR_CUDA;
        note(TPCONV_PHASE_BWD_EDGE_R, wn ? 2 : 1);
      }
    }
  }
  if (want_node) {
    for (int64_t s0 = 0; s0 < N; s0 += L.chunk_nodes) {
      const int nc = int(std::min<int64_t>(L.chunk_nodes, N - s0));
      {
        PhaseScope ps(TPCONV_PHASE_BWD_EDGE_S, s);
        const WorkList wl = work_list(L, workspace, 2, L.chunk_nodes);
        const int seg = piece_edges(N, E);
        if (build_work_list(wl, L, s_rowptr, int(s0), nc, seg, s)) return TPCONV_ERR_CUDA;
        if (TPC_WN_CALL_CPL(d, launch_wn_send, d, int(s0), nc, s_rowptr, perm, s_recv, edge_vec, g, S_, wl.extra,
                            wl.counter, seg, s))
          return TPCONV_ERR_CUDA;
        note(TPCONV_PHASE_BWD_EDGE_S, 3);  // list, two stream launches
      }
      {
        PhaseScope ps(TPCONV_PHASE_BWD_NODE_X, s);
        if (node_mix_sender(plan, L, workspace, int(s0), nc, S_, x, theta, tcp, dx, dtheta, s))
          return TPCONV_ERR_CUDA;
        const int64_t nx = channelwise(plan) ? cw_launches_in(d) : d.n_in;
        note(TPCONV_PHASE_BWD_NODE_X, int64_t(dx ? nx : 0) +
                                          int64_t(dtheta ? (channelwise(plan) ? nx : theta_gradient_launches(plan, L)) : 0));
      }
    }
  }
  return finish_call(plan, s, cudaSuccess);
}

int tpconv_double_backward(const tpconv_plan* plan, int64_t N, int64_t E, const int32_t* rowptr,
                           const int32_t* col, const int32_t* perm, const int32_t* s_rowptr,
                           const int32_t* s_recv, const float* edge_vec, const float* x, const float* theta,
                           const float* g, const float* gg_x, const float* gg_vec, const float* gg_theta,
                           float* d_g, float* d_x, float* d_vec, float* d_theta, void* workspace,
                           size_t workspace_bytes, void* stream) {
  if (!plan || N < 0 || E < 0) return TPCONV_ERR_INVALID_ARG;
  if (N > 0 && (!rowptr || !x || !theta || !g)) return TPCONV_ERR_INVALID_ARG;
  if (E > 0 && (!col || !edge_vec)) return TPCONV_ERR_INVALID_ARG;
  const bool want_node = d_x || d_theta;
  if (want_node && N > 0 && (!s_rowptr || (E > 0 && (!perm || !s_recv)))) return TPCONV_ERR_INVALID_ARG;
  WsLayout L;
  int st = check_ws(plan, TPCONV_OP_DOUBLE_BACKWARD, N, E, workspace, workspace_bytes, &L);
  if (st) return st;
  if ((st = ensure_device())) return st;
  const DevPlan& d = plan->dp;
  cudaStream_t s = S(stream);
  if (N > 0 && (st = validate_graph(plan, N, E, rowptr, col, edge_vec, s))) return st;
  const bool has_x1 = gg_x != nullptr, has_v = gg_vec != nullptr, has_t = gg_theta != nullptr;
  if (d_theta && cudaMemsetAsync(d_theta, 0, plan->theta_numel * 4, s)) return TPCONV_ERR_CUDA;
  if (d_x && N > 0 && cudaMemsetAsync(d_x, 0, size_t(N) * d.dim_in * 4, s)) return TPCONV_ERR_CUDA;
  if (N == 0) return finish(cudaSuccess);
  float* W0 = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.off_state);
  const int64_t Nc = L.chunk_nodes;
  float* treg = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.off_theta);
  float* gpack = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.off_pack);
  TcTheta tc0, tc1;
  const TcTheta* tc0p = nullptr;
  const TcTheta* tc1p = nullptr;
  if (use_tc(plan)) {
    PhaseScope ps(TPCONV_PHASE_OTHER, s);
    const bool wantR = d_vec && E > 0;
    if (prep_tc_theta(plan, TPCONV_OP_DOUBLE_BACKWARD, theta, treg, 0, d_g != nullptr, wantR, d_x != nullptr, &tc0, s)) return TPCONV_ERR_CUDA;
    tc0p = &tc0;
    if (has_t) {
      if (prep_tc_theta(plan, TPCONV_OP_DOUBLE_BACKWARD, gg_theta, treg, 1, d_g != nullptr, wantR, d_x != nullptr, &tc1, s))
        return TPCONV_ERR_CUDA;
      tc1p = &tc1;
    }
    note(TPCONV_PHASE_OTHER, (has_t ? 2 : 1) * tc_theta_launches(d, d_g != nullptr, wantR, d_x != nullptr));
  }
  // d_g = A1 . Theta + A0 . gg_theta
  if (d_g) {
    float* A1 = W0;
    float* A0 = W0 + size_t(Nc) * plan->a_floats;
    const float *t_hi = tc0p ? tc0.T_hi : nullptr, *t_lo = tc0p ? tc0.T_lo : nullptr;
    const float *gt_hi = tc1p ? tc1.T_hi : nullptr, *gt_lo = tc1p ? tc1.T_lo : nullptr;
    for (int64_t r0 = 0; r0 < N; r0 += Nc) {
      const int nc = int(std::min<int64_t>(Nc, N - r0));
      {
        PhaseScope ps(TPCONV_PHASE_DBL_EDGE_A, s);
        const WorkList wl = work_list(L, workspace, 0, L.chunk_nodes);
        const int seg = piece_edges(N, E);
        if (build_work_list(wl, L, rowptr, int(r0), nc, seg, s)) return TPCONV_ERR_CUDA;
        if (TPC_WN_CALL(d, launch_wn_dbla, d, int(r0), nc, rowptr, col, edge_vec, gg_vec, x, gg_x, A1,
                        has_t ? A0 : nullptr, wl.extra, wl.counter, seg, s))
          return TPCONV_ERR_CUDA;
        note(TPCONV_PHASE_DBL_EDGE_A, 3);  // list, two stream launches
      }
      PhaseScope ps(TPCONV_PHASE_DBL_NODE_A, s);
      if (node_mix_forward(plan, int(r0), nc, A1, theta, t_hi, t_lo, d_g, s, 0)) return TPCONV_ERR_CUDA;
      note(TPCONV_PHASE_DBL_NODE_A, d.n_out);
      if (has_t) {
        if (node_mix_forward(plan, int(r0), nc, A0, gg_theta, gt_hi, gt_lo, d_g, s, 1)) return TPCONV_ERR_CUDA;
        note(TPCONV_PHASE_DBL_NODE_A, d.n_out);
      }
    }
  }
  // d_vec from G = Theta^T g and Gt = gg_theta^T g
  if (d_vec && E > 0) {
    float* G = W0;
    float* Gt = W0 + size_t(Nc) * plan->a_floats;
    for (int64_t r0 = 0; r0 < N; r0 += Nc) {
      const int nc = int(std::min<int64_t>(Nc, N - r0));
      {
        PhaseScope ps(TPCONV_PHASE_OTHER, s);
        if (node_mix_adjoint(plan, int(r0), nc, g, theta, tc0p, gpack, G, s)) return TPCONV_ERR_CUDA;
        const int64_t na = channelwise(plan) ? cw_launches_out(d) : 2 * d.n_out;
        note(TPCONV_PHASE_OTHER, na);
        if (has_t) {
          if (node_mix_adjoint(plan, int(r0), nc, g, gg_theta, tc1p, gpack, Gt, s)) return TPCONV_ERR_CUDA;
          note(TPCONV_PHASE_OTHER, na);
        }
      }
      PhaseScope ps(TPCONV_PHASE_DBL_EDGE_R, s);
      const bool wn = d.wn_ok && aligned16(x) && aligned16(gg_x);
      const WorkList wl = work_list(L, workspace, 1, L.chunk_nodes);
      if (wn && build_work_list(wl, L, rowptr, int(r0), nc, kBatchEdges, s)) return TPCONV_ERR_CUDA;
      cudaError_t e = wn
                          ? TPC_WN_CALL(d, launch_wn_dadj, d, int(r0), nc, rowptr, col, edge_vec, gg_vec, x, gg_x, G,
                                        has_t ? Gt : nullptr, d_vec, wl.extra, wl.counter, s)
                          : TPC_RM_CALL(d.rm, launch_dbl_r_rm, d, int(r0), nc, rowptr, col, edge_vec, gg_vec, x,
                                        gg_x, G, has_t ? Gt : nullptr, d_vec, s);
      if (e) return TPCONV_ERR_CUDA;
      note(TPCONV_PHASE_DBL_EDGE_R, wn ? 2 : 1);
    }
  }
  // d_x = B1 . Theta + B0 . gg_theta ;  d_theta = x^T B1 + gg_x^T B0
  if (want_node) {
    float* B1 = W0;
    float* B0 = W0 + size_t(Nc) * plan->b_floats;
    for (int64_t s0 = 0; s0 < N; s0 += Nc) {
      const int nc = int(std::min<int64_t>(Nc, N - s0));
      {
        PhaseScope ps(TPCONV_PHASE_DBL_EDGE_S, s);
        float* B0u = (has_x1 || has_t) ? B0 : nullptr;
        const WorkList wl = work_list(L, workspace, 2, L.chunk_nodes);
        const int seg = piece_edges(N, E);
        if (build_work_list(wl, L, s_rowptr, int(s0), nc, seg, s)) return TPCONV_ERR_CUDA;
        if (TPC_WN_CALL(d, launch_wn_dbls, d, int(s0), nc, s_rowptr, perm, s_recv, edge_vec, gg_vec, g, B1, B0u,
                        wl.extra, wl.counter, seg, s))
          return TPCONV_ERR_CUDA;
        note(TPCONV_PHASE_DBL_EDGE_S, 3);  // list, two stream launches
      }
      PhaseScope ps(TPCONV_PHASE_DBL_NODE_X, s);
      float* dx1 = has_v ? d_x : nullptr;
      float* dt1 = has_v ? d_theta : nullptr;
      if (dx1 && node_mix_sender(plan, L, workspace, int(s0), nc, B1, x, theta, tc0p, dx1, nullptr, s))
        return TPCONV_ERR_CUDA;
      float* dx0 = has_t ? d_x : nullptr;
      float* dt0 = has_x1 ? d_theta : nullptr;
      if (dx0 && node_mix_sender(plan, L, workspace, int(s0), nc, B0, gg_x, gg_theta, tc1p, dx0, nullptr, s))
        return TPCONV_ERR_CUDA;
      // d_theta = x^T B1 + gg_x^T B0 in one pass
      if (dt1 || dt0) {
        const float *xa = dt1 ? x : nullptr, *Ba = dt1 ? B1 : nullptr;
        const float *xb = dt0 ? gg_x : nullptr, *Bb = dt0 ? B0 : nullptr;
        const cudaError_t e = channelwise(plan) ? cw_dtheta(d, int(s0), nc, xa, Ba, xb, Bb, d_theta, s)
                                                : theta_gradient(plan, L, workspace, int(s0), nc, xa, Ba, xb, Bb,
                                                                 d_theta, s);
        if (e) return TPCONV_ERR_CUDA;
      }
      const int64_t nx = channelwise(plan) ? cw_launches_in(d) : d.n_in;
      note(TPCONV_PHASE_DBL_NODE_X,
           int64_t(dx1 ? nx : 0) + int64_t(dx0 ? nx : 0) +
               ((dt1 || dt0) ? (channelwise(plan) ? nx : theta_gradient_launches(plan, L)) : 0));
    }
  }
  return finish_call(plan, s, cudaSuccess);
}

}  // extern "C"
