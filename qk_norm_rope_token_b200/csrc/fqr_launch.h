// fqr_launch.h -- host-side launch helpers shared by the entry points.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "fqr.h"
#include "fqr_device.cuh"

namespace fqr {

int launch_append(const fqr_append_params& p, cudaStream_t stream);
int launch_mla(const fqr_mla_params& p, cudaStream_t stream);

// Launch a persistent warp-task kernel: one block of kThreads per kWarps
// tasks, capped at the number of blocks that can be resident on the device at
// once (the kernel loops over the rest).  `launch(grid)` issues the <<<>>>.
template <class F>
int launch_persistent(const void* func, int64_t warp_tasks, size_t smem,
                      cudaStream_t /*stream*/, F&& launch) {
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FQR_ECUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return FQR_ECUDA;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return FQR_ECUDA;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, func, kThreads, smem) !=
          cudaSuccess ||
      per_sm < 1)
    return FQR_ECUDA;
  int64_t need = (warp_tasks + kWarps - 1) / kWarps;
  if (need < 1) need = 1;
  const int64_t cap = static_cast<int64_t>(per_sm) * sms;
  launch(static_cast<int>(need < cap ? need : cap));
  return cudaGetLastError() == cudaSuccess ? FQR_OK : FQR_ECUDA;
}

}  // namespace fqr
