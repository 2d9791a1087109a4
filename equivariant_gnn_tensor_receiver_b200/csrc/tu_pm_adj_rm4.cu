// Path-major lane-per-edge adjoint stream (first order), radial width 4.
#include "launch_pm.cuh"

namespace tpc {
template cudaError_t launch_adj_rm<4>(const DevPlan&, int, int, const int*, const int*, const float*, const float*,
                                       const float*, float*, float*, float*, cudaStream_t);
}  // namespace tpc
TPC_REGISTER_TU(pm_adj_rm4, &tpc::pm_adj_smem_rm<4>)
