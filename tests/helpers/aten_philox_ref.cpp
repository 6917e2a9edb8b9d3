// Independent Philox4x32-10 reference for the oracle pin: PyTorch's own
// header-only engine (ATen/core/PhiloxRNGEngine.h).  Reads lines
// "c0 c1 c2 c3 k0 k1" (decimal) from stdin, prints the four output words.
// The engine's offset is the counter's low 64 bits, its subsequence the high
// 64 bits, and its seed the 64-bit key.
#include <ATen/core/PhiloxRNGEngine.h>
#include <cstdint>
#include <cstdio>

int main() {
  unsigned long long c0, c1, c2, c3, k0, k1;
  while (std::scanf("%llu %llu %llu %llu %llu %llu", &c0, &c1, &c2, &c3, &k0, &k1) == 6) {
    uint64_t seed = (k1 << 32) | k0;
    uint64_t subseq = (c3 << 32) | c2;
    uint64_t offset = (c1 << 32) | c0;
    at::Philox4_32 eng(seed, subseq, offset);
    uint32_t w0 = eng(), w1 = eng(), w2 = eng(), w3 = eng();
    std::printf("%u %u %u %u\n", w0, w1, w2, w3);
  }
  return 0;
}
