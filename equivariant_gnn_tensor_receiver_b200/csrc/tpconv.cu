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
#include <cstring>
#include <mutex>

#include "gemm_simt.cuh"
#include "graph.cuh"
#include "launchers.h"
#include "plan.h"
#include "workspace.h"

using namespace tpc;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
bool g_ready[kMaxDevices];

// Once per device: upload the real-CG table and raise the kernels' shared memory
// limit.  The first call on a device synchronises it (cudaMemcpyToSymbol), so it
// must not happen inside a stream capture.
int ensure_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TPCONV_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_ready[dev]) return TPCONV_OK;
  const float* t = cg_table_f32();
  if (!t) return TPCONV_ERR_INTERNAL;
  if (upload_cg_fwd(t) || upload_cg_send(t) || upload_cg_radj(t)) return TPCONV_ERR_CUDA;
  if (radj_set_smem_limit(227 * 1024)) return TPCONV_ERR_CUDA;
  g_ready[dev] = true;
  return TPCONV_OK;
}

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

// out[r0 : r0+nc] = A . Theta  (per output block)
cudaError_t node_mix_forward(const DevPlan& d, int r0, int nc, const float* A, const float* theta, float* out,
                             cudaStream_t st) {
  for (int i3 = 0; i3 < d.n_out; ++i3) {
    const int n3 = 2 * d.out_l[i3] + 1, cout = d.out_mul[i3];
    const int p0 = first_path_of_out_block(d, i3);
    const float* th = theta + (p0 >= 0 ? d.path[p0].theta_off : 0);
    MView a = mrow(F(A) + size_t(nc) * d.a_pref[i3], d.Kb[i3]);
    MView b = mrow(F(th), cout);
    MView c = mview(out + size_t(r0) * d.dim_out + d.out_off[i3], n3, d.dim_out, 1, 1, n3, 0);
    cudaError_t e = gemm_simt(int64_t(nc) * n3, cout, d.Kb[i3], a, b, c, 0, st);
    if (e) return e;
  }
  return cudaSuccess;
}

// G[r0 : r0+nc] = g . Theta^T  (per output block)
cudaError_t node_mix_adjoint(const DevPlan& d, int r0, int nc, const float* g, const float* theta, float* G,
                             cudaStream_t st) {
  for (int i3 = 0; i3 < d.n_out; ++i3) {
    if (d.Kb[i3] == 0) continue;
    const int n3 = 2 * d.out_l[i3] + 1, cout = d.out_mul[i3];
    const int p0 = first_path_of_out_block(d, i3);
    MView a = mview(F(g) + size_t(r0) * d.dim_out + d.out_off[i3], n3, d.dim_out, 1, 1, n3, 0);
    MView b = mview(F(theta) + d.path[p0].theta_off, 1, 1, 0, 1, cout, 0);
    MView c = mrow(G + size_t(nc) * d.a_pref[i3], d.Kb[i3]);
    cudaError_t e = gemm_simt(int64_t(nc) * n3, d.Kb[i3], cout, a, b, c, 0, st);
    if (e) return e;
  }
  return cudaSuccess;
}

// dx[s0 : s0+nc] += B . Theta  and  dtheta += x^T B   (per path)
cudaError_t node_mix_sender(const DevPlan& d, int s0, int nc, const float* B, const float* x, const float* theta,
                            float* dx, float* dtheta, cudaStream_t st) {
  for (int p = 0; p < d.P; ++p) {
    const DevPath& q = d.path[p];
    const int n1 = 2 * q.l1 + 1;
    const int Kx = d.Kx[q.i1];
    MView bp = mrow(F(B) + size_t(nc) * d.b_pref[q.i1] + q.kxoff, Kx);
    cudaError_t e;
    if (dx) {
      MView th = mview(F(theta) + q.theta_off, q.c_out, int64_t(q.c_in) * q.c_out, 1, 1, q.c_out, 0);
      MView c = mview(dx + size_t(s0) * d.dim_in + q.in_off, n1, d.dim_in, 1, 1, n1, 0);
      if ((e = gemm_simt(int64_t(nc) * n1, q.c_in, int64_t(d.R) * q.c_out, bp, th, c, 1, st))) return e;
    }
    if (dtheta) {
      MView xa = mview(F(x) + size_t(s0) * d.dim_in + q.in_off, 1, n1, 0, n1, d.dim_in, 1);
      MView c = mview(dtheta + q.theta_off, 1, q.c_out, 0, q.c_out, int64_t(q.c_in) * q.c_out, 1);
      if ((e = gemm_simt(q.c_in, int64_t(d.R) * q.c_out, int64_t(nc) * n1, xa, bp, c, 2, st))) return e;
    }
  }
  return cudaSuccess;
}

int finish(cudaError_t e) {
  if (e != cudaSuccess) return TPCONV_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? TPCONV_OK : TPCONV_ERR_CUDA;
}

}  // namespace

extern "C" {

int tpconv_graph_transpose(const tpconv_plan* plan, int64_t N, int64_t E, const int32_t* rowptr,
                           const int32_t* col, int32_t* perm, int32_t* s_rowptr, int32_t* s_recv,
                           void* workspace, size_t workspace_bytes, void* stream) {
  if (!plan || N < 0 || E < 0) return TPCONV_ERR_INVALID_ARG;
  if (!s_rowptr || !rowptr || (E > 0 && (!col || !perm || !s_recv))) return TPCONV_ERR_INVALID_ARG;
  WsLayout L;
  int st = check_ws(plan, TPCONV_OP_TRANSPOSE, N, E, workspace, workspace_bytes, &L);
  if (st) return st;
  cudaStream_t s = S(stream);
  char* ws = static_cast<char*>(workspace);
  int* cnt = reinterpret_cast<int*>(ws + L.off_cursor);
  int* bsum = reinterpret_cast<int*>(ws + L.off_scan);
  int* tmp = reinterpret_cast<int*>(ws + L.off_tmp);
  if (cudaMemsetAsync(cnt, 0, size_t(N + 1) * 4, s)) return TPCONV_ERR_CUDA;
  if (E > 0) k_count_senders<<<1184, 256, 0, s>>>(E, col, cnt);
  const int64_t n = N + 1;  // scan N+1 counts (last is 0) so s_rowptr[N] = E
  const int nb = int((n + 1023) / 1024);
  k_scan_blocks<<<nb, 1024, 0, s>>>(n, cnt, s_rowptr, bsum);
  k_scan_totals<<<1, 1024, 0, s>>>(nb, bsum, bsum + nb);
  k_scan_add<<<nb, 1024, 0, s>>>(n, s_rowptr, bsum);
  if (E > 0) {
    if (cudaMemsetAsync(cnt, 0, size_t(N + 1) * 4, s)) return TPCONV_ERR_CUDA;
    k_fill_senders<<<1184, 128, 0, s>>>(N, rowptr, col, s_rowptr, cnt, tmp);
    k_sort_segments<<<2368, 256, 0, s>>>(N, rowptr, s_rowptr, tmp, perm, s_recv);
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
  float* A = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.off_state);
  for (int64_t r0 = 0; r0 < N; r0 += L.chunk_nodes) {
    const int nc = int(std::min<int64_t>(L.chunk_nodes, N - r0));
    if (launch_fwd_stream(d, int(r0), nc, rowptr, col, edge_vec, x, A, s)) return TPCONV_ERR_CUDA;
    cudaError_t e = node_mix_forward(d, int(r0), nc, A, theta, out, s);
    if (e) return TPCONV_ERR_CUDA;
  }
  return finish(cudaSuccess);
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
  if (dtheta && cudaMemsetAsync(dtheta, 0, plan->theta_numel * 4, s)) return TPCONV_ERR_CUDA;
  if (dx && N > 0 && cudaMemsetAsync(dx, 0, size_t(N) * d.dim_in * 4, s)) return TPCONV_ERR_CUDA;
  if (N == 0) return finish(cudaSuccess);
  float* S_ = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.off_state);
  if (want_edge && E > 0) {
    for (int64_t r0 = 0; r0 < N; r0 += L.chunk_nodes) {
      const int nc = int(std::min<int64_t>(L.chunk_nodes, N - r0));
      if (node_mix_adjoint(d, int(r0), nc, g, theta, S_, s)) return TPCONV_ERR_CUDA;
      if (launch_radj_stream(d, int(r0), nc, rowptr, col, edge_vec, x, S_, dvec, dY, db, s)) return TPCONV_ERR_CUDA;
    }
  }
  if (want_node) {
    for (int64_t s0 = 0; s0 < N; s0 += L.chunk_nodes) {
      const int nc = int(std::min<int64_t>(L.chunk_nodes, N - s0));
      if (launch_send_stream(d, int(s0), nc, s_rowptr, perm, s_recv, edge_vec, g, S_, s)) return TPCONV_ERR_CUDA;
      if (node_mix_sender(d, int(s0), nc, S_, x, theta, dx, dtheta, s)) return TPCONV_ERR_CUDA;
    }
  }
  return finish(cudaSuccess);
}

int tpconv_double_backward(const tpconv_plan* plan, int64_t N, int64_t E, const int32_t* rowptr,
                           const int32_t* col, const int32_t* perm, const int32_t* s_rowptr,
                           const int32_t* s_recv, const float* edge_vec, const float* x, const float* theta,
                           const float* g, const float* gg_x, const float* gg_vec, const float* gg_theta,
                           float* d_g, float* d_x, float* d_vec, float* d_theta, void* workspace,
                           size_t workspace_bytes, void* stream) {
  (void)plan; (void)N; (void)E; (void)rowptr; (void)col; (void)perm; (void)s_rowptr; (void)s_recv;
  (void)edge_vec; (void)x; (void)theta; (void)g; (void)gg_x; (void)gg_vec; (void)gg_theta; (void)d_g;
  (void)d_x; (void)d_vec; (void)d_theta; (void)workspace; (void)workspace_bytes; (void)stream;
  return TPCONV_ERR_UNSUPPORTED;
}

}  // extern "C"
