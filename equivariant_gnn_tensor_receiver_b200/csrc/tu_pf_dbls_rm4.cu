// Path-major node stream (dbls form), radial width 4.
#include "launch_pm.cuh"

namespace tpc {
template cudaError_t launch_dbl_s_rm<4>(const DevPlan&, int, int, const int*, const int*, const int*, const float*, const float*, const float*, float*, float*, cudaStream_t);
}  // namespace tpc
TPC_REGISTER_TU(pf_dbls_rm4, (&tpc::pf_smem_rm<4, false, true>))
