// fqr_runtime.cu -- host-side runtime of libfqr.so:
//   * a per-device cache of the launch facts every call needs (SM count,
//     shared-memory limits, resident blocks per kernel), so a call costs no
//     occupancy query after its first;
//   * the staged pipeline behind fqr_pipeline_* (include/fqr.h): pinned host
//     batches copied in, run and copied out on three streams, overlapped.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <new>
#include <vector>

#include "fqr.h"
#include "fqr_launch.h"

namespace fqr {

namespace {

struct OccKey {
  const void* fn;
  int threads;
  size_t smem;
  int dev;
  int per_sm;
};

std::mutex g_mu;
std::vector<DeviceInfo> g_dev;  // indexed by device ordinal
std::vector<OccKey> g_occ;

}  // namespace

int device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FQR_ECUDA;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (dev < static_cast<int>(g_dev.size()) && g_dev[dev].sms > 0) {
      *out = g_dev[dev];
      return FQR_OK;
    }
  }
  DeviceInfo d{dev, 0, 0, 0};
  if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&d.smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
          cudaSuccess)
    return FQR_ECUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (dev >= static_cast<int>(g_dev.size())) g_dev.resize(dev + 1, DeviceInfo{0, 0, 0, 0});
  g_dev[dev] = d;
  *out = d;
  return FQR_OK;
}

int resident_blocks(const void* fn, int threads, size_t smem, int* per_sm) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FQR_ECUDA;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    for (const OccKey& k : g_occ)
      if (k.fn == fn && k.threads == threads && k.smem == smem && k.dev == dev) {
        *per_sm = k.per_sm;
        return FQR_OK;
      }
  }
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return FQR_ECUDA;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, smem) != cudaSuccess || n < 1)
    return FQR_ECUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_occ.size() >= 4096) g_occ.clear();  // (bounded: distinct batch sizes give distinct keys)
  g_occ.push_back(OccKey{fn, threads, smem, dev, n});
  *per_sm = n;
  return FQR_OK;
}

}  // namespace fqr

// --------------------------------------------------------------- pipeline --

struct fqr_pipeline {
  int depth;
  int dev;
  std::vector<fqr_append_params> params;
  std::vector<void*> dev_in, dev_out;
  size_t in_bytes, out_bytes;
  cudaStream_t s_in, s_k, s_out;
  std::vector<cudaEvent_t> ev_in, ev_k, ev_out;
  std::vector<bool> used;
  int64_t next;
};

namespace {

void destroy_pipeline(fqr_pipeline* p) {
  if (p == nullptr) return;
  for (auto* v : {&p->ev_in, &p->ev_k, &p->ev_out})
    for (cudaEvent_t e : *v)
      if (e) cudaEventDestroy(e);
  for (cudaStream_t s : {p->s_in, p->s_k, p->s_out})
    if (s) cudaStreamDestroy(s);
  delete p;
}

}  // namespace

extern "C" {

int fqr_pipeline_create(int depth, const fqr_append_params* params, void* const* dev_in,
                        size_t in_bytes, void* const* dev_out, size_t out_bytes,
                        fqr_pipeline** out) {
  if (out == nullptr) return FQR_EINVAL;
  *out = nullptr;
  if (depth < 1 || depth > FQR_PIPELINE_MAX_DEPTH || params == nullptr || dev_in == nullptr ||
      dev_out == nullptr || in_bytes == 0 || out_bytes == 0)
    return FQR_EINVAL;
  for (int j = 0; j < depth; ++j) {
    if (dev_in[j] == nullptr || dev_out[j] == nullptr) return FQR_EINVAL;
    if (params[j].T == 0 && params[j].B == 0) return FQR_EINVAL;  // nothing to run
    const int rc = fqr::check_append(&params[j]);
    if (rc != FQR_OK) return rc;
  }
  fqr_pipeline* p = new (std::nothrow) fqr_pipeline();
  if (p == nullptr) return FQR_ECUDA;
  p->depth = depth;
  p->params.assign(params, params + depth);
  p->dev_in.assign(dev_in, dev_in + depth);
  p->dev_out.assign(dev_out, dev_out + depth);
  p->in_bytes = in_bytes;
  p->out_bytes = out_bytes;
  p->s_in = p->s_k = p->s_out = nullptr;
  p->ev_in.assign(depth, nullptr);
  p->ev_k.assign(depth, nullptr);
  p->ev_out.assign(depth, nullptr);
  p->used.assign(depth, false);
  p->next = 0;
  bool ok = cudaGetDevice(&p->dev) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p->s_in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p->s_k, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p->s_out, cudaStreamNonBlocking) == cudaSuccess;
  for (int j = 0; ok && j < depth; ++j)
    ok = cudaEventCreateWithFlags(&p->ev_in[j], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p->ev_k[j], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&p->ev_out[j], cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    (void)cudaGetLastError();
    destroy_pipeline(p);
    return FQR_ECUDA;
  }
  *out = p;
  return FQR_OK;
}

int fqr_pipeline_submit(fqr_pipeline* p, const void* host_in, void* host_out) {
  if (p == nullptr || host_in == nullptr || host_out == nullptr) return FQR_EINVAL;
  const int j = static_cast<int>(p->next % p->depth);
  // copy-in: once slot j's previous kernel has read its inputs
  if (p->used[j] && cudaStreamWaitEvent(p->s_in, p->ev_k[j], 0) != cudaSuccess) return FQR_ECUDA;
  if (cudaMemcpyAsync(p->dev_in[j], host_in, p->in_bytes, cudaMemcpyHostToDevice, p->s_in) !=
          cudaSuccess ||
      cudaEventRecord(p->ev_in[j], p->s_in) != cudaSuccess)
    return FQR_ECUDA;
  // kernel: after the copy-in, and once slot j's previous results are out
  if (cudaStreamWaitEvent(p->s_k, p->ev_in[j], 0) != cudaSuccess) return FQR_ECUDA;
  if (p->used[j] && cudaStreamWaitEvent(p->s_k, p->ev_out[j], 0) != cudaSuccess) return FQR_ECUDA;
  const int rc = fqr::launch_append(p->params[j], p->s_k);
  if (rc != FQR_OK) return rc;
  if (cudaEventRecord(p->ev_k[j], p->s_k) != cudaSuccess) return FQR_ECUDA;
  // copy-out
  if (cudaStreamWaitEvent(p->s_out, p->ev_k[j], 0) != cudaSuccess ||
      cudaMemcpyAsync(host_out, p->dev_out[j], p->out_bytes, cudaMemcpyDeviceToHost, p->s_out) !=
          cudaSuccess ||
      cudaEventRecord(p->ev_out[j], p->s_out) != cudaSuccess)
    return FQR_ECUDA;
  p->used[j] = true;
  ++p->next;
  return FQR_OK;
}

int fqr_pipeline_fork(fqr_pipeline* p, void* stream) {
  if (p == nullptr) return FQR_EINVAL;
  cudaEvent_t e;
  if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return FQR_ECUDA;
  bool ok = cudaEventRecord(e, static_cast<cudaStream_t>(stream)) == cudaSuccess;
  for (cudaStream_t s : {p->s_in, p->s_k, p->s_out})
    ok = ok && cudaStreamWaitEvent(s, e, 0) == cudaSuccess;
  cudaEventDestroy(e);  // (released once the waits resolve)
  return ok ? FQR_OK : FQR_ECUDA;
}

int fqr_pipeline_join(fqr_pipeline* p, void* stream) {
  if (p == nullptr) return FQR_EINVAL;
  // every submitted batch ends with its slot's copy-out, which follows its
  // kernel and copy-in; the last event of each used slot covers them all
  for (int j = 0; j < p->depth; ++j)
    if (p->used[j] &&
        cudaStreamWaitEvent(static_cast<cudaStream_t>(stream), p->ev_out[j], 0) != cudaSuccess)
      return FQR_ECUDA;
  return FQR_OK;
}

int fqr_pipeline_sync(fqr_pipeline* p) {
  if (p == nullptr) return FQR_EINVAL;
  for (cudaStream_t s : {p->s_in, p->s_k, p->s_out})
    if (cudaStreamSynchronize(s) != cudaSuccess) return FQR_ECUDA;
  return FQR_OK;
}

int fqr_pipeline_destroy(fqr_pipeline* p) {
  if (p == nullptr) return FQR_EINVAL;
  const int rc = fqr_pipeline_sync(p);
  destroy_pipeline(p);
  return rc;
}

}  // extern "C"
