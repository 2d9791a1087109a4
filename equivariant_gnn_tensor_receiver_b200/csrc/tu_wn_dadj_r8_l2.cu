// Warp-per-node stream (receiver adjoint, second order), radial width 8, feature degrees <= 2.
#include "launch_wn_adj.cuh"

TPC_WNA_TU(wn_dadj_r8_l2, dadj, 8, 2, true, const DevPlan&, int, int, const int*, const int*, const float*, const float*, const float*, const float*, const float*, const float*, float*, const int*, int*, cudaStream_t)
