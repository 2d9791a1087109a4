// Workspace layout of each operation (caller-provided device memory).
#pragma once

#include <cstddef>
#include <cstdint>

struct tpconv_plan;

namespace tpc {

struct WsLayout {
  size_t total;
  int64_t chunk_nodes;  // receivers (or senders) per chunk of node-side state
  size_t off_state, state_bytes;   // A / G / B state of one chunk
  size_t off_theta, theta_bytes;   // repacked Theta operands (2 slots x 6 regions)
  size_t off_pack, pack_bytes;     // one packed feature block of a chunk (tensor-core A operand)
  size_t off_cursor, off_scan, off_tmp;  // graph transpose scratch
  size_t off_lists, list_ints;     // work lists of the edge streams: kWorkLists x list_ints ints
};

// Work lists of one chunk (receiver pieces, receiver batches, sender pieces),
// each: a work counter (padded to 32 ints), the extra-item counts of the
// chunk's nodes and their exclusive scan (chunk_nodes + 1 ints each, padded),
// and the scan's block sums.
constexpr int kWorkLists = 3;
inline size_t work_list_pad(int64_t chunk_nodes) { return size_t(chunk_nodes + 1 + 31) & ~size_t(31); }
inline size_t work_list_ints(int64_t chunk_nodes) {
  const int64_t n = chunk_nodes + 1;
  return size_t(32 + 2 * work_list_pad(chunk_nodes) + (n + 1023) / 1024 + 2 + 63) & ~size_t(63);
}

int ws_layout(const tpconv_plan& p, int op, int64_t N, int64_t E, WsLayout* L);

}  // namespace tpc
