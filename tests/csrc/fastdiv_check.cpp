// Host check of fqr::FastDiv (the multiply-high division by invariant
// integers used by the kernels): for many divisors, every dividend in sampled
// ranges, including the ends of [0, 2^31), must divide exactly.
#include <cstdio>
#include <cstdint>
#include <random>
#include "fqr_device.cuh"

int main() {
  std::mt19937_64 rng(1234);
  uint64_t bad = 0, checked = 0;
  auto check = [&](uint32_t d, uint32_t n) {
    const fqr::FastDiv f(d);
    ++checked;
    if (f.div(n) != n / d || f.mod(n) != n % d) {
      if (bad < 5) std::printf("bad d=%u n=%u got %u want %u\n", d, n, f.div(n), n / d);
      ++bad;
    }
  };
  for (uint32_t d = 1; d <= 4096; ++d) {
    for (uint32_t n = 0; n < 20000; ++n) check(d, n);
    for (int k = 0; k < 2000; ++k) check(d, static_cast<uint32_t>(rng() % (1u << 31)));
    for (uint32_t n = (1u << 31) - 5000; n < (1u << 31); ++n) check(d, n);
  }
  for (int k = 0; k < 200000; ++k) {
    const uint32_t d = static_cast<uint32_t>(rng() % ((1u << 31) - 1)) + 1;
    check(d, static_cast<uint32_t>(rng() % (1u << 31)));
    check(d, (1u << 31) - 1);
    check(d, d - 1);
    check(d, d);
  }
  std::printf("checked=%llu bad=%llu\n", (unsigned long long)checked, (unsigned long long)bad);
  return bad ? 1 : 0;
}
