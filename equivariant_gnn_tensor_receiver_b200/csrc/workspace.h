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
};

int ws_layout(const tpconv_plan& p, int op, int64_t N, int64_t E, WsLayout* L);

}  // namespace tpc
