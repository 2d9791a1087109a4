// Warp-per-node stream (sender form, first order), radial width 16, feature degrees <= 3, 1 channel(s) per lane.
#include "launch_wn.cuh"

TPC_WN_TU_CPL(wn_send_r16_l3_c1, send, 16, 3, 1, false, false, const DevPlan&, int, int, const int*, const int*, const int*, const float*, const float*, float*, const int*, int*, int, cudaStream_t)
