// Fused backward sender stream, radial width 16.
#include "launch_fused.cuh"

namespace tpc {
template cudaError_t launch_send_rm<16>(const DevPlan&, int, int, const int*, const int*, const int*,
                                        const float*, const float*, float*, cudaStream_t);
}  // namespace tpc
TPC_REGISTER_TU(fused_send_rm16, &tpc::send_fused_smem_rm<16>)
