// Double-backward adjoint stream, radial width 8.
#include "launch_dbl.cuh"

namespace tpc {
template cudaError_t launch_dbl_r_rm<8>(const DevPlan&, int, int, const int*, const int*, const float*,
                                         const float*, const float*, const float*, const float*, const float*,
                                         float*, cudaStream_t);
}  // namespace tpc
TPC_REGISTER_TU(dbl_r_rm8, &tpc::dbl_r_smem_rm<8>)
