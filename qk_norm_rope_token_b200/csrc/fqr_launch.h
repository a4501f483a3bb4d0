// fqr_launch.h -- host-side launch helpers shared by the entry points.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "fqr.h"
#include "fqr_device.cuh"

namespace fqr {

struct HeadParams;
// Host-side argument checks of fqr_append_paged (FQR_OK or the error code).
int check_append(const fqr_append_params* p);
// The launch of fqr_append_paged on `stream`; with `plan` non-null, the plan
// of that launch instead (nothing is launched).
int launch_append(const fqr_append_params& p, cudaStream_t stream,
                  fqr_append_plan* plan = nullptr);
int launch_append_warp(const fqr_append_params& p, const HeadParams& hp, cudaStream_t stream,
                       fqr_append_plan* plan = nullptr);
// Warp tasks of the latency schedule for p, and how many warps of it the
// device holds at once (-1 if the runtime cannot tell).
int64_t latency_tasks(const fqr_append_params& p);
int64_t latency_capacity(const fqr_append_params& p);
// Threads per block the latency schedule uses for p (fqr_append_warp.cu).
int warp_block_threads(const fqr_append_params& p);
int launch_append_pipe(const fqr_append_params& p, const HeadParams& hp, cudaStream_t stream,
                       fqr_append_plan* plan = nullptr);
int launch_mla(const fqr_mla_params& p, cudaStream_t stream);

// Launch facts of the current device, cached after the first query
// (fqr_runtime.cu).
struct DeviceInfo {
  int dev, sms, smem_optin, smem_sm;
};
int device_info(DeviceInfo* out);
// Resident blocks per SM of kernel fn at this block size and dynamic shared
// memory (raising the kernel's dynamic shared-memory limit when smem > 48 KiB),
// cached per (kernel, threads, smem, device).
int resident_blocks(const void* fn, int threads, size_t smem, int* per_sm);

// Launch `kernel(args)` on `stream` with programmatic stream serialization,
// so that it may begin while the preceding kernel in the stream finishes; the
// kernel itself waits (griddepcontrol.wait) before reading any input.
// cluster > 1: the grid is launched as thread-block clusters of that many
// blocks (grid a multiple of it).
template <class Args>
int launch_pdl(void (*kernel)(const Args), int grid, int threads, size_t smem,
               cudaStream_t stream, const Args& args, int cluster = 1) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(cluster);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cluster > 1 ? 2 : 1;
  if (cudaLaunchKernelEx(&cfg, kernel, args) != cudaSuccess) {
    (void)cudaGetLastError();
    return FQR_ECUDA;
  }
  return cudaGetLastError() == cudaSuccess ? FQR_OK : FQR_ECUDA;
}

// Launch a persistent warp-task kernel: one block of `threads` per
// threads / 32 tasks, capped at the number of blocks that can be resident on
// the device at once (the kernel loops over the rest).  `launch(grid)` issues
// the <<<>>>.
template <class F>
int launch_persistent(const void* func, int64_t warp_tasks, size_t smem,
                      cudaStream_t /*stream*/, F&& launch, int threads = kThreads) {
  DeviceInfo d;
  int per_sm = 0;
  if (device_info(&d) != FQR_OK || resident_blocks(func, threads, smem, &per_sm) != FQR_OK)
    return FQR_ECUDA;
  const int warps = threads / 32;
  int64_t need = (warp_tasks + warps - 1) / warps;
  if (need < 1) need = 1;
  const int64_t cap = static_cast<int64_t>(per_sm) * d.sms;
  return launch(static_cast<int>(need < cap ? need : cap));
}

}  // namespace fqr
