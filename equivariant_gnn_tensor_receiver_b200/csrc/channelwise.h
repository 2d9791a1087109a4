// Node-level contractions of the channel-wise operator family
// (W_e[p] = diag(sum_k b_k Theta[p][k, :]), Theta[p] of shape R x C).
//
// The edge streams build the same node-side states as for the full family:
//   A[(r, m3), koff_p + k C + u]   receiver state (sum_e b_ek T_e[p, u, m3])
//   G[(r, m3), koff_p + k C + u]   its cotangent
//   B[(s, m1), kxoff_p + k C + w]  sender state
// and only the maps between these states and the features change: with one
// weight per channel, every contraction over C_in (or C_out) becomes a
// per-channel sum over (p, k).  All four are HBM-bound.
#pragma once

#include <cuda_runtime.h>

#include "plan.h"

namespace tpc {

// out[r0 + n, i3, u, m3] (= mode 0, += mode 1) sum_{p -> i3} sum_k Theta[p][k][u] A_i3[(n, m3), koff_p + k C + u]
cudaError_t cw_forward(const DevPlan& d, int r0, int nc, const float* A, const float* theta, float* out, int mode,
                       cudaStream_t st);

// G_i3[(n, m3), koff_p + k C + u] = Theta[p][k][u] g[r0 + n, i3, u, m3]
cudaError_t cw_adjoint(const DevPlan& d, int r0, int nc, const float* g, const float* theta, float* G,
                       cudaStream_t st);

// dx[s0 + n, i1, u, m1] += sum_{p from i1} sum_k Theta[p][k][u] B_i1[(n, m1), kxoff_p + k C + u]
cudaError_t cw_dx(const DevPlan& d, int s0, int nc, const float* B, const float* theta, float* dx, cudaStream_t st);

// dTheta[p][k][u] += sum_n sum_m1 xa[s0 + n, i1, u, m1] Ba_i1[(n, m1), kxoff_p + k C + u]
//                    (+ the same for xb, Bb when given)
cudaError_t cw_dtheta(const DevPlan& d, int s0, int nc, const float* xa, const float* Ba, const float* xb,
                      const float* Bb, float* dtheta, cudaStream_t st);

// kernel launches of cw_forward / cw_adjoint (per call), of cw_dx / cw_dtheta (per call)
int cw_launches_out(const DevPlan& d);
int cw_launches_in(const DevPlan& d);

}  // namespace tpc
