// Path-major lane-per-edge adjoint stream (second order), radial width 8.
#include "launch_pm.cuh"

namespace tpc {
template cudaError_t launch_dadj_rm<8>(const DevPlan&, int, int, const int*, const int*, const float*,
                                        const float*, const float*, const float*, const float*, const float*, float*,
                                        cudaStream_t);
}  // namespace tpc
TPC_REGISTER_TU(pm_dadj_rm8, &tpc::pm_dadj_smem_rm<8>)
