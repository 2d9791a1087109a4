// Allocation-free forward: tpconv_forward with its workspace in a fixed device
// array of this library instead of memory the caller provides.
//
// Some callers cannot allocate device memory for the workspace:
//   * a C or C++ host program that links only this library and has no device
//     allocator of its own;
//   * a plugin inside a host framework that owns device memory through its own
//     caching allocator, which the plugin may not bypass;
//   * a fixed-latency loop that must not call cudaMalloc / cudaFree, which can
//     synchronise the device.
// tpconv_forward_static serves them from a file-scope __device__ array of
// TPCONV_STATIC_SCRATCH_BYTES.  Its device address is looked up with
// cudaGetSymbolAddress on every call (a host-side query, no device work), so a
// context that was reset and re-created never sees a stale address; nothing
// here allocates.
//
// No part of the scratch has to start at zero: the forward writes every region
// of its workspace (node state, tensor-core operands of Theta, packed output
// rows) before it reads it, so stale contents of an earlier call are harmless.
//
// All calls share the one array per device: calls whose executions overlap (on
// different streams, or from several host threads) race on it and must be
// serialised by the caller, e.g. by issuing them on one stream.
#include <cuda_runtime.h>

#include "../../include/tpconv.h"

namespace {

static __device__ __align__(256) unsigned char g_scratch[TPCONV_STATIC_SCRATCH_BYTES];

// device address of g_scratch in the current device's context.  The host-side
// symbol g_scratch is only a handle: code on the host must never dereference it
// or pass it to a kernel, only the address returned here.
int scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return TPCONV_ERR_CUDA;
  *out = p;
  return TPCONV_OK;
}

}  // namespace

extern "C" int tpconv_forward_static(const tpconv_plan* plan, int64_t N, int64_t E, const int32_t* rowptr,
                                     const int32_t* col, const float* edge_vec, const float* x,
                                     const float* theta, float* out, void* stream) {
  if (!plan) return TPCONV_ERR_INVALID_ARG;
  size_t need = 0;
  int st = tpconv_workspace_size(plan, TPCONV_OP_FORWARD, N, E, &need);
  if (st != TPCONV_OK) return st;
  if (need > size_t(TPCONV_STATIC_SCRATCH_BYTES)) return TPCONV_ERR_WORKSPACE_TOO_SMALL;
  void* ws = nullptr;
  if ((st = scratch_address(&ws)) != TPCONV_OK) return st;
  return tpconv_forward(plan, N, E, rowptr, col, edge_vec, x, theta, out, ws, size_t(TPCONV_STATIC_SCRATCH_BYTES),
                        stream);
}
