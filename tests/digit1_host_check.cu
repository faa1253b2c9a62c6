// Host check of the selection's digit-1 map (the __host__ __device__ functions of the library's
// common header): every bin's smallest key maps to it, the key before the next bin's smallest
// key maps to it, bins rise with the key, and a bin that claims a shared key prefix has one.
// Prints "bad <count>" and then, for each top-15-bit value t, the bin of the keys t << 17 and
// (t << 17) | 0x1FFFF as little-endian uint16 pairs on stdout (after a newline).
#include <cstdint>
#include <cstdio>

#include "../top_retrieval_attention_b200/csrc/common.cuh"

int main() {
  using namespace ra;
  long bad = 0;
  for (uint32_t b = 0; b < 2048; ++b) {
    const unsigned long long f = digit1_floor(b), g = digit1_floor(b + 1);
    if (g <= f) ++bad;
    if (digit1_bin(static_cast<uint32_t>(f)) != b) ++bad;
    if (digit1_bin(static_cast<uint32_t>(g - 1)) != b) ++bad;
    const int pb = digit1_prefix_bits(b);
    if (pb > 0 && (f >> (32 - pb)) != ((g - 1) >> (32 - pb))) ++bad;
  }
  uint32_t prev = 0;
  for (unsigned long long k = 0; k < (1ull << 32); k += 65521) {
    const uint32_t bb = digit1_bin(static_cast<uint32_t>(k));
    if (bb < prev) ++bad;
    prev = bb;
  }
  std::printf("bad %ld\n", bad);
  for (uint32_t t = 0; t < 32768; ++t) {
    const uint16_t lo = static_cast<uint16_t>(digit1_bin(t << 17));
    const uint16_t hi = static_cast<uint16_t>(digit1_bin((t << 17) | 0x1FFFFu));
    std::fwrite(&lo, 2, 1, stdout);
    std::fwrite(&hi, 2, 1, stdout);
  }
  return bad != 0;
}
