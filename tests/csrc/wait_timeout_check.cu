// A bounded wait that runs out, on purpose, in a test build with a 50 ms
// budget: block 0 waits on an mbarrier that nothing arrives at, gives up and
// reports through fqr::flag_timeout; block 1 first writes the flags as a
// valid call's prologue does (0).  Checks that the kernel returns within a
// few seconds, that every flag then reads kFlagTimeout (-2), and that the
// context is still usable (a second launch and a copy succeed).  No fault,
// trap or hang: the wait ends on the globaltimer budget.
#define FQR_WAIT_LIMIT_NS 50000000ull
#include <chrono>
#include <cstdint>
#include <cstdio>
#include "fqr_device.cuh"

__global__ void wait_forever(int32_t* flags, int B, int* result) {
  __shared__ uint64_t bar;
  if (blockIdx.x > 0) {  // a valid call's flag stores
    for (int b = threadIdx.x; b < B; b += blockDim.x) flags[b] = 0;
    return;
  }
  if (threadIdx.x == 0) {
    fqr::mbar_init(&bar, 1);
    fqr::mbar_init_fence();
  }
  __syncthreads();
  const bool done = fqr::mbar_wait(&bar, 0);  // no thread ever arrives
  if (threadIdx.x < 32 && !done) fqr::flag_timeout(flags, B, threadIdx.x);
  if (threadIdx.x == 0) *result = done ? 1 : 0;
}

int main() {
  const int B = 100;
  int32_t* flags = nullptr;
  int* result = nullptr;
  if (cudaMalloc(&flags, B * sizeof(int32_t)) != cudaSuccess ||
      cudaMalloc(&result, sizeof(int)) != cudaSuccess)
    return 2;
  cudaMemset(flags, 0x5A, B * sizeof(int32_t));
  cudaMemset(result, 0x7F, sizeof(int));
  const auto t0 = std::chrono::steady_clock::now();
  wait_forever<<<2, 64>>>(flags, B, result);
  const cudaError_t e = cudaDeviceSynchronize();
  const double s = std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count();
  int32_t h[B];
  int r = -1;
  if (e != cudaSuccess || cudaMemcpy(h, flags, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(&r, result, sizeof r, cudaMemcpyDeviceToHost) != cudaSuccess) {
    printf("CUDA error: %s\n", cudaGetErrorString(e));
    return 1;
  }
  int bad = 0;
  for (int b = 0; b < B; ++b) bad += h[b] != fqr::kFlagTimeout;
  // the context is still usable
  wait_forever<<<1, 32>>>(flags, 0, result);
  const bool usable = cudaDeviceSynchronize() == cudaSuccess;
  printf("wait gave up: %s, flags not -2: %d, %.3f s, context usable: %s\n", r == 0 ? "yes" : "no",
         bad, s, usable ? "yes" : "no");
  return (r == 0 && bad == 0 && s > 0.04 && s < 5.0 && usable) ? 0 : 1;
}
