// GPU checks of the payload divisions against IEEE division (__fdiv_rn).
// fqr::div2_bounded (dynamic Q), in the domain the kernel uses it in,
// |a / b| <= 448 (a dynamic-Q payload never exceeds upper_max <= 448):
//   (1) bit-for-bit equal quotients whenever a = +-0, or |a| >= 2^-100 and
//       the IEEE quotient is not subnormal (Markstein's correction is exact
//       when nothing underflows);
//   (2) equal E4M3 codes (RN, satfinite) for every a.
// fqr::divide_pairs (K / V: 16 values of a lane by one scale d, any values):
//   (3) equal E4M3 codes for every value, whichever way the guard goes.
//   usage: division_check all <divisor bits hex> | rand <seed> <n>
//          | kvall <scale bits hex> | kvrand <seed> <n>
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
  const bool in_bits =
      bounded && (a == 0.0f || (fabsf(a) >= 0x1p-100f && fabsf(ref) >= 0x1p-126f));
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
__device__ __forceinline__ uint32_t code(float x) { return fqr::pack_e4m3x2(x, x) & 0xFF; }
// every binary32 value a as all 16 values of a lane (the guard sees |a|)
__global__ void kv_all(uint32_t dbits, uint64_t base) {
  const float d = __uint_as_float(dbits);
  const uint64_t i = base + (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const float a = __uint_as_float((uint32_t)i);
  float2 y[8];
  for (int j = 0; j < 8; ++j) y[j] = make_float2(a, a);
  fqr::divide_pairs(y, d);
  const uint32_t ref = code(__fdiv_rn(a, d));
  if (code(y[0].x) != ref || code(y[7].y) != ref) {
    if (atomicAdd(&g_bad_code, 1ull) == 0) {
      g_first_a = __float_as_uint(a);
      g_first_b = dbits;
    }
  }
}
// 16 random bit patterns per lane (mixed magnitudes, so the guard goes either
// way) and a random scale: positive normal with exponent in [-100, 100], or
// any bit pattern one time in eight
__global__ void kv_rand(uint64_t seed, uint64_t base) {
  const uint64_t i = base + (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const uint64_t h = mix(seed ^ mix(i));
  const uint32_t db = (uint32_t)(h >> 32);
  const uint32_t dbits = (h & 7) == 0 ? db : (((uint32_t)(27 + (db % 201)) << 23) | (db & 0x7FFFFF));
  const float d = __uint_as_float(dbits);
  float2 y[8], x[8];
  for (int j = 0; j < 8; ++j) {
    const uint64_t v = mix(h + 0x51ull * (j + 1));
    // mostly moderate values (exponent field 90..160), some raw patterns
    const uint32_t lo = (uint32_t)v, hi = (uint32_t)(v >> 32);
    const uint32_t ex = 90 + (lo >> 25) % 71;
    x[j].x = __uint_as_float((v & 0xF00) == 0 ? lo : ((lo & 0x807FFFFFu) | (ex << 23)));
    x[j].y = __uint_as_float((v & 0xF000) == 0 ? hi : ((hi & 0x807FFFFFu) | ((90 + (hi >> 25) % 71) << 23)));
    y[j] = x[j];
  }
  fqr::divide_pairs(y, d);
  for (int j = 0; j < 8; ++j) {
    if (code(y[j].x) != code(__fdiv_rn(x[j].x, d)) || code(y[j].y) != code(__fdiv_rn(x[j].y, d))) {
      if (atomicAdd(&g_bad_code, 1ull) == 0) {
        g_first_a = __float_as_uint(x[j].x);
        g_first_b = dbits;
      }
    }
  }
}
int main(int argc, char** argv) {
  if (argc < 3) return 2;
  const int threads = 256;
  const uint64_t chunk = 1ull << 30;
  if (!strcmp(argv[1], "all")) {
    const uint32_t bbits = (uint32_t)strtoul(argv[2], nullptr, 16);
    for (uint64_t base = 0; base < (1ull << 32); base += chunk)
      all_dividends<<<(unsigned)(chunk / threads), threads>>>(bbits, base);
  } else if (!strcmp(argv[1], "kvall")) {
    const uint32_t dbits = (uint32_t)strtoul(argv[2], nullptr, 16);
    for (uint64_t base = 0; base < (1ull << 32); base += chunk)
      kv_all<<<(unsigned)(chunk / threads), threads>>>(dbits, base);
  } else if (!strcmp(argv[1], "kvrand")) {
    const uint64_t seed = strtoull(argv[2], nullptr, 10), n = strtoull(argv[3], nullptr, 10);
    for (uint64_t base = 0; base < n; base += chunk)
      kv_rand<<<(unsigned)(chunk / threads), threads>>>(seed, base);
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
