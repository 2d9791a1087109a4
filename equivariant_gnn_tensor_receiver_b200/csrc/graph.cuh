// Sender-sorted view of a receiver-CSR graph (once per graph): a counting sort
// of the edges by sender, made deterministic by sorting every sender segment by
// edge id.  Used by the transposed (sender-sorted) backward stream.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "plan.h"

namespace tpc {

__global__ void k_count_senders(int64_t E, const int* __restrict__ col, int* __restrict__ cnt) {
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < E; e += int64_t(gridDim.x) * blockDim.x)
    atomicAdd(&cnt[col[e]], 1);
}

// exclusive scan, 1024 elements per block; block totals to bsum
__global__ void __launch_bounds__(1024) k_scan_blocks(int64_t n, const int* __restrict__ in,
                                                      int* __restrict__ out, int* __restrict__ bsum) {
  __shared__ int s[1024];
  const int64_t i = blockIdx.x * 1024LL + threadIdx.x;
  int v = i < n ? in[i] : 0;
  s[threadIdx.x] = v;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {
    int t = threadIdx.x >= o ? s[threadIdx.x - o] : 0;
    __syncthreads();
    s[threadIdx.x] += t;
    __syncthreads();
  }
  if (i < n) out[i] = s[threadIdx.x] - v;
  if (threadIdx.x == 1023) bsum[blockIdx.x] = s[1023];
}

// in-place exclusive scan of the block totals (single block, any count)
__global__ void __launch_bounds__(1024) k_scan_totals(int nb, int* __restrict__ bsum, int* __restrict__ total) {
  __shared__ int s[1024];
  __shared__ int carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < nb; base += 1024) {
    const int i = base + threadIdx.x;
    int v = i < nb ? bsum[i] : 0;
    s[threadIdx.x] = v;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
      int t = threadIdx.x >= o ? s[threadIdx.x - o] : 0;
      __syncthreads();
      s[threadIdx.x] += t;
      __syncthreads();
    }
    if (i < nb) bsum[i] = carry + s[threadIdx.x] - v;
    __syncthreads();
    if (threadIdx.x == 1023) carry += s[1023];
    __syncthreads();
  }
  if (threadIdx.x == 0) *total = carry;
}

__global__ void k_scan_add(int64_t n, int* __restrict__ out, const int* __restrict__ bsum) {
  const int64_t i = blockIdx.x * 1024LL + threadIdx.x;
  if (i < n) out[i] += bsum[blockIdx.x];
}

// scatter each edge into its sender's segment (arbitrary order inside a segment)
__global__ void k_fill_senders(int64_t N, const int* __restrict__ rowptr, const int* __restrict__ col,
                               const int* __restrict__ s_rowptr, int* __restrict__ cursor,
                               int* __restrict__ tmp) {
  for (int64_t r = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; r < N; r += int64_t(gridDim.x) * blockDim.x) {
    for (int e = rowptr[r]; e < rowptr[r + 1]; ++e) {
      const int s = col[e];
      const int pos = atomicAdd(&cursor[s], 1);
      tmp[s_rowptr[s] + pos] = e;
    }
  }
}

// one warp per sender: rank sort of its (distinct) edge ids, then the receiver
// of each edge by binary search in rowptr
__global__ void k_sort_segments(int64_t N, const int* __restrict__ rowptr, const int* __restrict__ s_rowptr,
                                const int* __restrict__ tmp, int* __restrict__ perm, int* __restrict__ s_recv) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  for (int64_t s = blockIdx.x * int64_t(blockDim.x >> 5) + (threadIdx.x >> 5); s < N; s += warps) {
    const int j0 = s_rowptr[s], j1 = s_rowptr[s + 1];
    for (int a = j0 + lane; a < j1; a += 32) {
      const int v = tmp[a];
      int rank = 0;
      for (int b = j0; b < j1; ++b) rank += tmp[b] < v;
      perm[j0 + rank] = v;
      int lo = 0, hi = int(N);  // largest r with rowptr[r] <= v
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (rowptr[mid] <= v) lo = mid;
        else hi = mid;
      }
      s_recv[j0 + rank] = lo;
    }
  }
}

}  // namespace tpc

namespace tpc {

// ---- work lists of the edge streams -----------------------------------------
// Node i of a chunk owns work item i (its first piece); a node whose CSR segment
// is longer than `seg` edges owns extra items, one per further piece.  One CTA
// of 1024 threads writes extra[i] = the first extra item of node i (exclusive
// scan of the extra counts, in rounds of 1024 with a carry), extra[nc] = their
// total, and resets the streams' work counter.
__global__ void __launch_bounds__(1024) k_build_work_list(int nc, const int* __restrict__ ptr, int n0, int seg,
                                                          int* __restrict__ extra, int* __restrict__ counter) {
  __shared__ int s[1024];
  __shared__ int carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base <= nc; base += 1024) {
    const int i = base + threadIdx.x;
    int c = 0;
    if (i < nc) {
      const int deg = ptr[n0 + i + 1] - ptr[n0 + i];
      c = deg > seg ? (deg + seg - 1) / seg - 1 : 0;
    }
    s[threadIdx.x] = c;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
      const int t = threadIdx.x >= o ? s[threadIdx.x - o] : 0;
      __syncthreads();
      s[threadIdx.x] += t;
      __syncthreads();
    }
    if (i <= nc) extra[i] = carry + s[threadIdx.x] - c;
    __syncthreads();
    if (threadIdx.x == 1023) carry += s[1023];
    __syncthreads();
  }
  if (threadIdx.x == 0) *counter = 0;
}

}  // namespace tpc
