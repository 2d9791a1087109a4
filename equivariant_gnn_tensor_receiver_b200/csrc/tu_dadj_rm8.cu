// Lane-per-edge double-backward adjoint stream, radial width 8.
#include "launch_dadj.cuh"
#include "launch_streams.cuh"

namespace tpc {
template cudaError_t launch_dadj_rm<8>(const DevPlan&, int, int, const int*, const int*, const float*,
                                        const float*, const float*, const float*, const float*, const float*,
                                        float*, cudaStream_t);
}  // namespace tpc
TPC_REGISTER_TU(dadj_rm8, &tpc::dadj_smem_rm<8>)
