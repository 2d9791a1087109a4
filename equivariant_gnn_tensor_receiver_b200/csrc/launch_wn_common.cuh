// Grid helpers shared by the launchers of the warp-per-node edge streams.
#pragma once

#include <cuda_runtime.h>

#include "launchers.h"
#include "wn_layout.h"

namespace tpc {

// path-major grid of the first pieces (channel-lane streams)
inline unsigned wn_grid_pm(const DevPlan& d, int nc) { return unsigned(d.P) * unsigned((nc + kWnWarps - 1) / kWnWarps); }
// persistent grid: as many CTAs as fit on the device at once
template <class K>
unsigned wn_grid(K kernel, int smem) {
  int dev = 0, sms = 148, per = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, kernel, 32 * kWnWarps, smem) != cudaSuccess || per < 1)
    per = 1;
  return unsigned(sms * per);
}

}  // namespace tpc
