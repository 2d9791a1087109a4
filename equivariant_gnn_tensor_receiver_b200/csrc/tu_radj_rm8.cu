// Receiver adjoint stream, radial width 8.
#include "launch_streams.cuh"

namespace tpc {
template cudaError_t launch_radj_rm<8>(const DevPlan&, int, int, const int*, const int*, const float*,
                                        const float*, const float*, float*, float*, float*, cudaStream_t);
}  // namespace tpc
TPC_REGISTER_TU(radj_rm8, &tpc::radj_smem_rm<8>)
