// Fused forward receiver stream, radial width 4.
#include "launch_fused.cuh"

namespace tpc {
template cudaError_t launch_fwd_rm<4>(const DevPlan&, int, int, const int*, const int*, const float*,
                                       const float*, float*, cudaStream_t);
}  // namespace tpc
TPC_REGISTER_TU(fused_fwd_rm4, &tpc::fwd_fused_smem_rm<4>)
