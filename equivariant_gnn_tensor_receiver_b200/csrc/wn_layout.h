// Shared-memory layout of the warp-per-node edge streams (host and device).
//
// A warp owns one node: it walks the node's CSR segment and keeps every partial
// sum of that node (lane = channel) or of its edges (lane = edge) in registers,
// so the streams need no block-wide barrier and no cross-warp reduction.  Each
// warp has its own slice of dynamic shared memory, laid out below in floats.
#pragma once

#if defined(__CUDACC__)
#define TPC_HD __host__ __device__
#else
#define TPC_HD
#endif

namespace tpc {

constexpr int kWnWarps = 4;   // warps (nodes) per CTA
constexpr int kWnSub = 4;     // edges per staged sub-batch of the channel-lane streams
constexpr int kWnChunk = 4;   // channels per staged chunk of the edge-lane (adjoint) streams

// ---- lane = channel (receiver / sender forms, first and second order) ------
// M, Md : coupling matrices of the 32 edges of the current geometry batch, nmp floats each
// B, Bd : their radial bases, RM floats each
// X, X1 : two sub-batch buffers of kWnSub staged neighbour rows, xs floats per row
struct WnLay {
  int M, Md, B, Bd, X, X1;
  int nmp, xs, buf;  // buf = floats of one X buffer
  int total;         // floats per warp
};

TPC_HD inline WnLay wn_layout_of(int RM, int cpl, int nimax, int nmz_max, bool dbl, bool two_src) {
  WnLay L;
  L.nmp = (nmz_max + 3) & ~3;
  L.xs = (32 * cpl * nimax + 3) & ~3;
  L.buf = kWnSub * L.xs;
  L.M = 0;
  L.Md = L.M + 32 * L.nmp;
  L.B = L.Md + (dbl ? 32 * L.nmp : 0);
  L.Bd = L.B + 32 * RM;
  L.X = L.Bd + (dbl ? 32 * RM : 0);
  L.X1 = L.X + 2 * L.buf;
  L.total = L.X1 + (two_src ? 2 * L.buf : 0);
  return L;
}
TPC_HD inline int wn_smem_bytes(int RM, int cpl, int nimax, int nmz_max, bool dbl, bool two_src) {
  return kWnWarps * wn_layout_of(RM, cpl, nimax, nmz_max, dbl, two_src).total * 4;
}

// ---- lane = edge (receiver adjoint streams, first and second order) --------
// Second order: a warp's lanes are 32 consecutive CSR edges, which may belong
// to several receivers; the G rows of up to `ns` of them are staged at once (a
// window spanning more receivers runs its channel loop once per group of ns).
// First order: a warp's lanes are up to 32 edges of one receiver (one slot).
// G, Gt : two chunk buffers, each ns slots of kWnChunk channels of one
//         receiver's G (and Gt, only with the gg_Theta operand),
//         [u][k/2][m3][k&1] with row stride RM * (2 l3 + 1) of the path (zero
//         where never staged); slot stride gslot = kWnChunk * gs + 4 floats, so
//         that lanes reading different slots fall into different bank quads
// X, X1 : two chunk buffers of the 32 lanes' rows, [lane][u * n1 + m1] with row
//         stride xs, xs / 4 odd: the 16-byte reads of 8 consecutive lanes fall
//         into distinct bank quads
// Geo   : per lane Y[16], b[RM] (and Yd[16], bd[RM]), odd stride
// Acc   : per lane accumulators that persist across paths (dY, or wY and hY), odd stride
// XZ    : one row of zeros (xs floats); a lane whose receiver is not in the group
//         being staged reads it for its x rows (and any staged G slot), which
//         makes every term it adds zero.
//
// ns: 1 for the first order; for the second order 2 with the Gt operand, else
// 3 when the slices of three slots still let two CTAs share an SM (the same
// rule on host and device), else 2.
constexpr int kWnaTwoCtaBytes = (228 * 1024 - 2 * 1024) / 2;  // dynamic shared memory of one of two CTAs per SM
struct WnaLay {
  int G, Gt, X, X1, XZ, Geo, Acc;
  int ns, gs, gslot, gbuf, xs, xbuf, geos, accs;
  int total;
};

TPC_HD inline WnaLay wna_layout_of(int RM, int n3max, int n1max, bool dbl, bool gt) {
  WnaLay L;
  L.gs = RM * n3max;
  L.gslot = kWnChunk * L.gs + 4;
  L.xs = (kWnChunk * n1max + 3) & ~3;
  if ((L.xs >> 2) % 2 == 0) L.xs += 4;
  L.xbuf = 32 * L.xs;
  L.geos = (dbl ? 2 : 1) * (16 + RM) + 1;
  L.accs = (dbl ? 32 : 16) + 1;
  for (int ns = dbl ? (gt ? 2 : 3) : 1;; --ns) {
    L.ns = ns;
    L.gbuf = ns * L.gslot;
    L.G = 0;
    L.Gt = L.G + 2 * L.gbuf;
    L.X = L.Gt + (gt ? 2 * L.gbuf : 0);
    L.X1 = L.X + 2 * L.xbuf;
    L.XZ = L.X1 + (dbl ? 2 * L.xbuf : 0);
    L.Geo = L.XZ + L.xs;
    L.Acc = L.Geo + 32 * L.geos;
    L.total = (L.Acc + 32 * L.accs + 3) & ~3;
    if (ns <= 2 || kWnWarps * L.total * 4 + 16 <= kWnaTwoCtaBytes) break;
  }
  return L;
}
// the warps' slices and one int (the CTA's batch count)
TPC_HD inline int wna_smem_bytes(int RM, int n3max, int n1max, bool dbl, bool gt) {
  return kWnWarps * wna_layout_of(RM, n3max, n1max, dbl, gt).total * 4 + 16;
}

// ---- work items of the streams (lists built in graph.cuh) ----
// Item t < nc is node t's first piece; item t >= nc is extra piece t - nc.
constexpr int kBatchEdges = 32;  // edges per adjoint work item (lane = edge): 32 consecutive CSR edges

#if defined(__CUDACC__)
// item t >= nc: the extra piece u = t - nc belongs to the node i with extra[i] <= u < extra[i+1]
__device__ __forceinline__ int extra_owner(const int* __restrict__ extra, int nc, int u) {
  int lo = 0, hi = nc;  // extra[lo] <= u < extra[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (extra[mid] <= u) lo = mid;
    else hi = mid;
  }
  return lo;
}

#endif

}  // namespace tpc
