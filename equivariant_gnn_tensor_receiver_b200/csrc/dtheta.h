// Theta gradient of the streaming schedule (dtheta.cu).
#pragma once

#include <cuda_runtime.h>

#include "plan.h"

namespace tpc {

// dtheta[p][k][u][w] += sum over nodes s0 .. s0+nc-1 of the chunk and m1 of
// xa[s, u, m1] * Ba[s, k, w, m1]  (+ the same with xb, Bb when both are given).
// Ba / Bb: the chunk's sender-state buffers ([block i1][node * (2l1+1) + m1][Kx]);
// xa / xb: full node feature arrays [N][dim_in].  dtheta must be zeroed once
// before the first chunk; partial sums are added atomically.
cudaError_t dtheta_accumulate(const DevPlan& d, int s0, int nc, const float* xa, const float* Ba, const float* xb,
                              const float* Bb, float* dtheta, cudaStream_t st);
// raises the kernel's dynamic shared-memory limit (once per device)
cudaError_t dtheta_smem_init();

}  // namespace tpc
