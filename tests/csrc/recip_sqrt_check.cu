// GPU check of fqr::rn_recip_sqrt -- the inverse RMS's 1 / sqrt(v) with the
// definition's two roundings, RN(1 / RN(sqrt(v))) -- against CUDA's correctly
// rounded __frcp_rn(__fsqrt_rn(v)) on every binary32 input (NaN results
// compare equal to NaN).  Prints the number of mismatches and the first one;
// exits 1 if there is any.
#include <cstdint>
#include <cstdio>
#include "fqr_device.cuh"

__device__ unsigned long long g_bad;
__device__ unsigned int g_first;
__device__ unsigned long long g_hist[256];  // mismatches by the input's exponent field

__global__ void sweep(uint64_t base) {
  const uint64_t i = base + (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const float v = __uint_as_float((uint32_t)i);
  const float got = fqr::rn_recip_sqrt(v), want = __frcp_rn(__fsqrt_rn(v));
  const bool same = (isnan(got) && isnan(want)) || __float_as_uint(got) == __float_as_uint(want);
  if (!same) {
    if (atomicAdd(&g_bad, 1ull) == 0) g_first = (uint32_t)i;
    atomicAdd(&g_hist[((uint32_t)i >> 23) & 0xFF], 1ull);
  }
}

int main() {
  const uint64_t chunk = 1ull << 28;
  for (uint64_t base = 0; base < (1ull << 32); base += chunk) {
    sweep<<<(unsigned)(chunk / 256), 256>>>(base);
    if (cudaGetLastError() != cudaSuccess) return 2;
  }
  unsigned long long bad = 0;
  unsigned int first = 0;
  if (cudaMemcpyFromSymbol(&bad, g_bad, sizeof bad) != cudaSuccess) return 2;
  if (cudaMemcpyFromSymbol(&first, g_first, sizeof first) != cudaSuccess) return 2;
  unsigned long long hist[256];
  if (cudaMemcpyFromSymbol(hist, g_hist, sizeof hist) != cudaSuccess) return 2;
  printf("rn_recip_sqrt: %llu mismatches of 2^32", bad);
  if (bad) printf(" (first input bits %08x)", first);
  printf("\n");
  for (int e = 0; e < 256; ++e)
    if (hist[e]) printf("  exponent field %d (2^%d): %llu\n", e, e - 127, hist[e]);
  return bad ? 1 : 0;
}
