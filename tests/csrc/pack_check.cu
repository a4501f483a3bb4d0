// Every binary32 input through the kernels' packed encoders, against the CPU
// oracle's encoders (the format definitions: BF16 round to nearest even; E4M3
// round to nearest even, saturating at +-448, NaN -> 0x7F).  The kernels'
// fqr::pack_e4m3x2 (cvt.rn.satfinite.e4m3x2.f32) and fqr::pack_bf16x2
// (cvt.rn.bf16x2.f32) encode chunks of inputs on the GPU, in both halves of
// the packed pair; host threads compare each code with the oracle's.  BF16
// NaN results compare equal to NaN (the payload is not part of the format's
// rounding).  Prints the mismatch counts and the first mismatching input of
// each format; exits 1 if there is any.
#include <cstdint>
#include <cstdio>
#include <thread>
#include <vector>

#include "fqr_device.cuh"
extern "C" {
#include "fqr_oracle.h"
}

__device__ unsigned long long g_pair_bad;  // the two halves of a pair disagree

__global__ void encode(uint64_t base, uint32_t n, uint8_t* e4m3, uint16_t* bf16) {
  const uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const uint32_t bits = (uint32_t)(base + i);
  const float v = __uint_as_float(bits);
  const float u = __uint_as_float(bits ^ 0x5A5A5A5Au);  // a partner value in the other half
  const uint32_t e_lo = fqr::pack_e4m3x2(v, u), e_hi = fqr::pack_e4m3x2(u, v);
  const uint32_t b_lo = fqr::pack_bf16x2(v, u), b_hi = fqr::pack_bf16x2(u, v);
  const uint16_t b0 = (uint16_t)(b_lo & 0xFFFF), b1 = (uint16_t)(b_hi >> 16);
  const bool nan0 = (b0 & 0x7FFF) > 0x7F80, nan1 = (b1 & 0x7FFF) > 0x7F80;
  if ((e_lo & 0xFF) != ((e_hi >> 8) & 0xFF) || !(b0 == b1 || (nan0 && nan1)))
    atomicAdd(&g_pair_bad, 1ull);
  e4m3[i] = (uint8_t)(e_lo & 0xFF);
  bf16[i] = b0;
}

static bool bf16_nan(uint16_t c) { return (c & 0x7FFF) > 0x7F80; }

int main() {
  const uint32_t chunk = 1u << 26;
  uint8_t* d8 = nullptr;
  uint16_t* d16 = nullptr;
  if (cudaMalloc(&d8, chunk) != cudaSuccess || cudaMalloc(&d16, 2ull * chunk) != cudaSuccess)
    return 2;
  std::vector<uint8_t> h8(chunk);
  std::vector<uint16_t> h16(chunk);
  const unsigned nt = std::thread::hardware_concurrency() ? std::thread::hardware_concurrency() : 4;
  uint64_t bad8 = 0, bad16 = 0;
  uint32_t first8 = 0, first16 = 0;
  for (uint64_t base = 0; base < (1ull << 32); base += chunk) {
    encode<<<chunk / 256, 256>>>(base, chunk, d8, d16);
    if (cudaMemcpy(h8.data(), d8, chunk, cudaMemcpyDeviceToHost) != cudaSuccess) return 2;
    if (cudaMemcpy(h16.data(), d16, 2ull * chunk, cudaMemcpyDeviceToHost) != cudaSuccess) return 2;
    std::vector<uint64_t> b8(nt, 0), b16(nt, 0);
    std::vector<uint32_t> f8(nt, 0), f16(nt, 0);
    std::vector<std::thread> th;
    for (unsigned t = 0; t < nt; ++t) {
      th.emplace_back([&, t] {
        for (uint32_t i = t; i < chunk; i += nt) {
          const uint32_t bits = (uint32_t)(base + i);
          float v;
          memcpy(&v, &bits, 4);
          const uint8_t w8 = fqro_f32_to_e4m3_rn_satfinite(v);
          const uint16_t w16 = fqro_f32_to_bf16_rne(v);
          if (h8[i] != w8 && b8[t]++ == 0) f8[t] = bits;
          const bool ok16 = h16[i] == w16 || (bf16_nan(h16[i]) && bf16_nan(w16));
          if (!ok16 && b16[t]++ == 0) f16[t] = bits;
        }
      });
    }
    for (auto& x : th) x.join();
    for (unsigned t = 0; t < nt; ++t) {
      if (b8[t] && !bad8) first8 = f8[t];
      if (b16[t] && !bad16) first16 = f16[t];
      bad8 += b8[t];
      bad16 += b16[t];
    }
  }
  cudaFree(d8);
  cudaFree(d16);
  unsigned long long pair_bad = 0;
  if (cudaMemcpyFromSymbol(&pair_bad, g_pair_bad, sizeof pair_bad) != cudaSuccess) return 2;
  printf("low / high half disagreements: %llu\n", pair_bad);
  printf("pack_e4m3x2: %llu mismatches of 2^32", (unsigned long long)bad8);
  if (bad8) printf(" (first input bits %08x)", first8);
  printf("\npack_bf16x2: %llu mismatches of 2^32", (unsigned long long)bad16);
  if (bad16) printf(" (first input bits %08x)", first16);
  printf("\n");
  return (bad8 || bad16 || pair_bad) ? 1 : 0;
}
