// Warp-per-node stream (sender form, second order), radial width 16, feature degrees <= 3.
#include "launch_wn.cuh"

TPC_WN_TU(wn_dbls_r16_l3, dbls, 16, 3, false, true, const DevPlan&, int, int, const int*, const int*, const int*, const float*, const float*, const float*, float*, float*, const int*, int*, int, cudaStream_t)
