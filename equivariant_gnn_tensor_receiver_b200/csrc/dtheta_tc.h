// Theta gradient on the tensor cores (dtheta_tc.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "plan.h"

namespace tpc {

// The tensor-core Theta gradient serves the plan's shapes (full family, every
// B-block column offset a multiple of four floats, c_in <= 256).  Host-only
// shape check, the same on every machine (workspace sizes depend on it).
bool dtheta_tc_shape_ok(const DevPlan& d);
// column tile (>= the largest c_in): 32, 64, 128 or 256
int dtheta_tc_bn(const DevPlan& d);
// workspace floats: packed x of a chunk of nc nodes (2 pairs x {hi, lo}), and
// the partial tiles of one call
size_t dtheta_tc_xt_floats(const DevPlan& d, int64_t nc);
size_t dtheta_tc_partial_floats(const DevPlan& d);

// dtheta[p][k][u][w] += sum over nodes s0 .. s0+nc-1 and m1 of
// xa[s, u, m1] * Ba[(s, m1), kxoff(p) + k c_out + w]  (+ the same with xb, Bb).
// Ba / Bb: the chunk's sender-state buffers; xa / xb: full [N][dim_in] arrays.
// xt, partial: workspace of dtheta_tc_xt_floats / dtheta_tc_partial_floats.
// split: 3xTF32 (fp32 accuracy), else one TF32 pass.  Deterministic: partial
// tiles are summed in a fixed order, no atomics.  wait_ns bounds every wait of
// the kernel on its own pipeline; an expired wait is recorded (read with
// dtheta_tc_read_error) and the call's result is then not valid.
cudaError_t dtheta_tc_accumulate(const DevPlan& d, int s0, int nc, const float* xa, const float* Ba,
                                 const float* xb, const float* Bb, float* dtheta, float* xt, float* partial,
                                 bool split, uint64_t wait_ns, cudaStream_t st);

// per-context set-up: dynamic shared-memory limits of the kernels
cudaError_t dtheta_tc_init();
// first error code recorded by an expired wait since the last read (0 = none); clears it
cudaError_t dtheta_tc_read_error(int* code);

}  // namespace tpc
