// Receiver adjoint stream, radial width 16.
#include "launch_streams.cuh"

namespace tpc {
template cudaError_t launch_radj_rm<16>(const DevPlan&, int, int, const int*, const int*, const float*,
                                        const float*, const float*, float*, float*, float*, cudaStream_t);
}  // namespace tpc
TPC_REGISTER_TU(radj_rm16, &tpc::radj_smem_rm<16>)
