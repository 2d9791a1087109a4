// Shared-memory layout of the path-major adjoint streams (host and device).
#pragma once

namespace tpc {

constexpr int kPmWarps = 8;   // warps per CTA; they split a path's channels
constexpr int kPmBatch = 32;  // edges per batch (lane = edge)

// Float offsets.  tile = channels staged per step (also the G row stride);
// dbl adds the second G / x buffers of the double backward.
struct PmLay {
  int Y, Yd, B, Bd, S, G, Gt, X, X1, Red;
  int xs;    // staged row stride (odd: conflict-free lane-per-row reads)
  int tile;
};

#if defined(__CUDACC__)
#define TPC_HD __host__ __device__
#else
#define TPC_HD
#endif

TPC_HD inline PmLay pm_layout_of(int RM, int tile, int n3max, int n1max, int R, bool dbl) {
  PmLay L;
  L.tile = tile;
  L.Y = 0;
  L.Yd = L.Y + kPmBatch * 16;
  L.B = L.Yd + kPmBatch * 16;
  L.Bd = L.B + kPmBatch * RM;
  L.S = L.Bd + kPmBatch * RM;
  L.G = (L.S + kPmBatch + 3) & ~3;
  const int g = R * n3max * tile;
  L.Gt = L.G + g;
  L.X = L.Gt + (dbl ? g : 0);
  L.xs = (tile * n1max) | 1;
  L.X1 = L.X + kPmBatch * L.xs;
  L.Red = L.X1 + (dbl ? kPmBatch * L.xs : 0);
  return L;
}

TPC_HD inline int pm_smem_bytes(int RM, int tile, int n3max, int n1max, int R, bool dbl) {
  const PmLay L = pm_layout_of(RM, tile, n3max, n1max, R, dbl);
  return (L.Red + kPmWarps * kPmBatch * (dbl ? 32 + 2 * RM : 16 + RM)) * 4;
}

}  // namespace tpc
