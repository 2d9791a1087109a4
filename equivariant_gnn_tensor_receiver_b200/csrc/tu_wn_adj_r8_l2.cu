// Warp-per-node stream (receiver adjoint, first order), radial width 8, feature degrees <= 2.
#include "launch_wn_adj.cuh"

TPC_WNA_TU(wn_adj_r8_l2, adj, 8, 2, false, const DevPlan&, int, int, const int*, const int*, const float*, const float*, const float*, float*, float*, float*, const int*, int*, cudaStream_t)
