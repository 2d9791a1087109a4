// Lane-per-edge receiver adjoint stream, radial width 8.
#include "launch_adj.cuh"
#include "launch_streams.cuh"

namespace tpc {
template cudaError_t launch_adj_rm<8>(const DevPlan&, int, int, const int*, const int*, const float*,
                                       const float*, const float*, float*, float*, float*, cudaStream_t);
}  // namespace tpc
TPC_REGISTER_TU(adj_rm8, &tpc::adj_smem_rm<8>)
