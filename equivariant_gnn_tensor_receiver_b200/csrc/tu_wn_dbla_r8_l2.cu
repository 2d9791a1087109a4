// Warp-per-node stream (receiver form, second order), radial width 8, feature degrees <= 2.
#include "launch_wn.cuh"

TPC_WN_TU(wn_dbla_r8_l2, dbla, 8, 2, true, true, const DevPlan&, int, int, const int*, const int*, const float*, const float*, const float*, const float*, float*, float*, const int*, int*, int, cudaStream_t)
