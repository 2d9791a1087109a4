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
  size_t off_theta, theta_bytes;   // repacked Theta operands (theta_region below)
  size_t off_pack, pack_bytes;     // one packed feature block of a chunk (tensor-core A operand)
  size_t off_cursor, off_scan, off_tmp;  // graph transpose scratch
  size_t off_lists, list_ints;     // work lists of the edge streams: kWorkLists x list_ints ints
  size_t off_xt, xt_bytes;         // tensor-core Theta gradient: packed x of a chunk (2 pairs x {hi, lo})
  size_t off_part, part_bytes;     // tensor-core Theta gradient: partial tiles of one call
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

// Repacked Theta operands of the tensor-core contractions.  The region holds
// slices of theta_numel floats (rounded up to 64) indexed by (slot, kind, half):
// slot 0 = Theta, 1 = gg_Theta; kind 0 = T (per output block Theta_blk^T),
// 1 = N (Theta split elementwise), 2 = X (per input block [C_in][K_x]);
// half 0 = hi, 1 = lo (3xTF32 only).  Each operation reserves what it uses:
//   forward: slot 0, T;  backward: slot 0, N and X;  double backward: both
//   slots, T, N and X.
// Plans whose Theta contractions do not run on tensor cores reserve none.
enum ThetaKind { kThetaT = 0, kThetaN = 1, kThetaX = 2 };
inline int theta_kinds_mask(int op) { return op == 0 ? 1 : op == 1 ? 6 : op == 2 ? 7 : 0; }
inline int theta_slots(int op) { return op == 2 ? 2 : (op == 0 || op == 1) ? 1 : 0; }
inline int theta_region_count(int op, bool tc, bool split) {
  if (!tc) return 0;
  const int m = theta_kinds_mask(op);
  const int nk = (m & 1) + ((m >> 1) & 1) + ((m >> 2) & 1);
  return theta_slots(op) * nk * (split ? 2 : 1);
}
// index of a slice, or -1 when the operation does not reserve it
inline int theta_region(int op, int slot, int kind, int half, bool tc, bool split) {
  const int m = theta_kinds_mask(op);
  if (!tc || slot >= theta_slots(op) || !((m >> kind) & 1) || (half && !split)) return -1;
  int kpos = 0, nk = 0;
  for (int k = 0; k < 3; ++k)
    if ((m >> k) & 1) {
      if (k < kind) ++kpos;
      ++nk;
    }
  const int nh = split ? 2 : 1;
  return (slot * nk + kpos) * nh + half;
}

}  // namespace tpc
