// Path-major node stream (fwd form), radial width 4.
#include "launch_pm.cuh"

namespace tpc {
template cudaError_t launch_fwd_rm<4>(const DevPlan&, int, int, const int*, const int*, const float*, const float*, float*, cudaStream_t);
}  // namespace tpc
TPC_REGISTER_TU(pf_fwd_rm4, (&tpc::pf_smem_rm<4, true, false>))
