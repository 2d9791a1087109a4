// Warp-per-node stream (receiver form, first order), radial width 8, feature degrees <= 2, 2 channel(s) per lane.
#include "launch_wn.cuh"

TPC_WN_TU_CPL(wn_fwd_r8_l2_c2, fwd, 8, 2, 2, true, false, const DevPlan&, int, int, const int*, const int*, const float*, const float*, float*, const int*, int*, int, cudaStream_t)
