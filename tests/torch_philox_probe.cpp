// Independent Philox4x32-10: PyTorch's header-only CPU engine, called (not copied) to
// cross-check the oracle's Philox words.  Reads lines "c0 c1 c2 c3 k0 k1" (decimal) on stdin,
// prints the four output words of each block in decimal.
#include <ATen/core/PhiloxRNGEngine.h>
#include <cstdint>
#include <cstdio>

int main() {
  unsigned long long c[4], k[2];
  while (std::scanf("%llu %llu %llu %llu %llu %llu", &c[0], &c[1], &c[2], &c[3], &k[0], &k[1]) == 6) {
    uint64_t seed = (uint64_t)k[0] | ((uint64_t)k[1] << 32);
    uint64_t subsequence = (uint64_t)c[2] | ((uint64_t)c[3] << 32);
    uint64_t offset = (uint64_t)c[0] | ((uint64_t)c[1] << 32);
    at::philox_engine eng(seed, subsequence, offset);
    uint32_t w0 = eng(), w1 = eng(), w2 = eng(), w3 = eng();
    std::printf("%u %u %u %u\n", w0, w1, w2, w3);
  }
  return 0;
}
