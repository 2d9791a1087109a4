// Path-major node stream (dbla form), radial width 8.
#include "launch_pm.cuh"

namespace tpc {
template cudaError_t launch_dbl_a_rm<8>(const DevPlan&, int, int, const int*, const int*, const float*, const float*, const float*, const float*, float*, float*, cudaStream_t);
}  // namespace tpc
TPC_REGISTER_TU(pf_dbla_rm8, (&tpc::pf_smem_rm<8, true, true>))
