// Path-major node stream (fwd form), radial width 8.
#include "launch_pm.cuh"

namespace tpc {
template cudaError_t launch_fwd_rm<8>(const DevPlan&, int, int, const int*, const int*, const float*, const float*, float*, cudaStream_t);
}  // namespace tpc
TPC_REGISTER_TU(pf_fwd_rm8, (&tpc::pf_smem_rm<8, true, false>))
