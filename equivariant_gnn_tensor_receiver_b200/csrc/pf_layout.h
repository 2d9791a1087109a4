// Shared-memory layout of the path-major node streams (host and device).
#pragma once

#include "pm_layout.h"

namespace tpc {

constexpr int kPfGeoMax = 128;  // edges whose geometry a node CTA caches
constexpr int kPfRedChunk = 40;  // partial-state floats per lane reduced per round

// shared layout of one node CTA (floats): cached geometry of the node's first
// kPfGeoMax edges (recomputed per batch beyond), the batch's gathered rows of
// one block (and of a second source), the batch's coupling matrices, and the
// reduction buffer.
struct PfLay {
  int Y, Yd, B, Bd, S, X, X1, M, Md, Red;
  int xs;  // staged row stride (multiple of 4)
};

TPC_HD inline PfLay pf_layout_of(int RM, int nmax, int nmz_max, bool dbl) {
  PfLay L;
  constexpr int G = kPfGeoMax + kPmBatch;  // cached slots + one scratch batch
  L.Y = 0;
  L.Yd = L.Y + G * 16;
  L.B = L.Yd + G * 16;
  L.Bd = L.B + G * RM;
  L.S = L.Bd + G * RM;
  L.xs = 32 * nmax + 4;
  L.X = (L.S + G + 3) & ~3;
  L.X1 = L.X + kPmBatch * L.xs;
  const int nm = (nmz_max + 3) & ~3;
  L.M = L.X1 + (dbl ? kPmBatch * L.xs : 0);
  L.Md = L.M + kPmBatch * nm;
  L.Red = L.Md + (dbl ? kPmBatch * nm : 0);
  return L;
}
TPC_HD inline int pf_smem_bytes(int RM, int nmax, int nmz_max, bool dbl) {
  const PfLay L = pf_layout_of(RM, nmax, nmz_max, dbl);
  return (L.Red + kPmWarps * kPfRedChunk * 32) * 4;
}

}  // namespace tpc
