// Warp-per-node stream (receiver form, second order), radial width 4, feature degrees <= 3.
#include "launch_wn.cuh"

TPC_WN_TU(wn_dbla_r4_l3, dbla, 4, 3, true, true, const DevPlan&, int, int, const int*, const int*, const float*, const float*, const float*, const float*, float*, float*, const int*, int*, int, cudaStream_t)
