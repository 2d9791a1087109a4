// Warp-per-node stream (receiver adjoint, second order), radial width 8, feature degrees <= 3.
#include "launch_wn_adj.cuh"

TPC_WNA_TU(wn_dadj_r8_l3, dadj, 8, 3, true, const DevPlan&, int, int, const int*, const int*, const float*, const float*, const float*, const float*, const float*, const float*, float*, const int*, int*, cudaStream_t)
