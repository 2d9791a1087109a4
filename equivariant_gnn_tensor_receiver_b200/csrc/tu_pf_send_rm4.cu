// Path-major node stream (send form), radial width 4.
#include "launch_pm.cuh"

namespace tpc {
template cudaError_t launch_send_rm<4>(const DevPlan&, int, int, const int*, const int*, const int*, const float*, const float*, float*, cudaStream_t);
}  // namespace tpc
TPC_REGISTER_TU(pf_send_rm4, (&tpc::pf_smem_rm<4, false, false>))
