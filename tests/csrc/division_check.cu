// GPU check of fqr::div2_bounded (the dynamic-Q payload division) against
// IEEE division (__fdiv_rn):
// in the domain the kernel uses it in, |a / b| <= 448 (a dynamic-Q payload
// never exceeds upper_max <= 448):
//   (1) bit-for-bit equal quotients whenever |a| >= 2^-100 or a = +-0;
//   (2) equal E4M3 codes (RN, satfinite) for every a.
//   usage: division_check all <divisor bits hex> | rand <seed> <n>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include "fqr_head.cuh"

__device__ unsigned long long g_bad_bits, g_bad_code;
__device__ unsigned int g_first_a, g_first_b;

__device__ __forceinline__ bool same(float x, float y) {
  if (isnan(x) && isnan(y)) return true;
  return __float_as_uint(x) == __float_as_uint(y);
}
__device__ __forceinline__ void check(float a, float b, float r) {
  const float q = fqr::div2_bounded(make_float2(a, a), make_float2(b, b), make_float2(r, r)).x;
  const float ref = __fdiv_rn(a, b);
  const bool bounded = !isnan(a) && fabsf(ref) <= 448.0f;
  const bool in_bits = bounded && (fabsf(a) >= 0x1p-100f || a == 0.0f);
  if (in_bits && !same(q, ref)) {
    if (atomicAdd(&g_bad_bits, 1ull) == 0) {
      g_first_a = __float_as_uint(a);
      g_first_b = __float_as_uint(b);
    }
  }
  if (bounded) {
    if ((fqr::pack_e4m3x2(q, q) & 0xFF) != (fqr::pack_e4m3x2(ref, ref) & 0xFF))
      atomicAdd(&g_bad_code, 1ull);
  }
}
__global__ void all_dividends(uint32_t bbits, uint64_t base) {
  const float b = __uint_as_float(bbits), r = __frcp_rn(b);
  const uint64_t i = base + (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  check(__uint_as_float((uint32_t)i), b, r);
}
__device__ __forceinline__ uint64_t mix(uint64_t x) {  // splitmix64 finaliser
  x += 0x9E3779B97F4A7C15ull;
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  return x ^ (x >> 31);
}
// divisors of the dynamic-scale form: positive normals in [2^-30, 2^100]
__global__ void random_pairs(uint64_t seed, uint64_t base) {
  const uint64_t i = base + (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const uint64_t h = mix(seed ^ mix(i));
  const uint32_t abits = (uint32_t)h, bb = (uint32_t)(h >> 32);
  const uint32_t bbits = ((uint32_t)(97 + (bb % 131)) << 23) | (bb & 0x7FFFFF);
  const float b = __uint_as_float(bbits);
  check(__uint_as_float(abits), b, __frcp_rn(b));
}
int main(int argc, char** argv) {
  if (argc < 3) return 2;
  const int threads = 256;
  const uint64_t chunk = 1ull << 30;
  if (!strcmp(argv[1], "all")) {
    const uint32_t bbits = (uint32_t)strtoul(argv[2], nullptr, 16);
    for (uint64_t base = 0; base < (1ull << 32); base += chunk)
      all_dividends<<<(unsigned)(chunk / threads), threads>>>(bbits, base);
  } else {
    const uint64_t seed = strtoull(argv[2], nullptr, 10), n = strtoull(argv[3], nullptr, 10);
    for (uint64_t base = 0; base < n; base += chunk)
      random_pairs<<<(unsigned)(chunk / threads), threads>>>(seed, base);
  }
  if (cudaDeviceSynchronize() != cudaSuccess) { printf("cuda error\n"); return 3; }
  unsigned long long bb = 0, bc = 0;
  unsigned int fa = 0, fb = 0;
  cudaMemcpyFromSymbol(&bb, g_bad_bits, sizeof bb);
  cudaMemcpyFromSymbol(&bc, g_bad_code, sizeof bc);
  cudaMemcpyFromSymbol(&fa, g_first_a, sizeof fa);
  cudaMemcpyFromSymbol(&fb, g_first_b, sizeof fb);
  printf("bit_mismatches=%llu code_mismatches=%llu first=0x%08x/0x%08x\n", bb, bc, fa, fb);
  return (bb || bc) ? 1 : 0;
}
