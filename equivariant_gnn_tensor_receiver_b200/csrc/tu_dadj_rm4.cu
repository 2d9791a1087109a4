// Lane-per-edge double-backward adjoint stream, radial width 4.
#include "launch_dadj.cuh"
#include "launch_streams.cuh"

namespace tpc {
template cudaError_t launch_dadj_rm<4>(const DevPlan&, int, int, const int*, const int*, const float*,
                                        const float*, const float*, const float*, const float*, const float*,
                                        float*, cudaStream_t);
}  // namespace tpc
TPC_REGISTER_TU(dadj_rm4, &tpc::dadj_smem_rm<4>)
