// Double-backward receiver and sender streams, radial width 4.
#include "launch_dbl.cuh"

namespace tpc {
template cudaError_t launch_dbl_a_rm<4>(const DevPlan&, int, int, const int*, const int*, const float*,
                                         const float*, const float*, const float*, float*, float*, cudaStream_t);
template cudaError_t launch_dbl_s_rm<4>(const DevPlan&, int, int, const int*, const int*, const int*,
                                         const float*, const float*, const float*, float*, float*, cudaStream_t);
}  // namespace tpc
TPC_REGISTER_TU(dbl_as_rm4, nullptr)
