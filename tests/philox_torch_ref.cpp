// Independent Philox4x32-10 for the oracle's pin: PyTorch's open-source
// at::Philox4_32 engine (ATen/core/PhiloxRNGEngine.h). Reads lines of
// "ctr0 ctr1 ctr2 ctr3 key0 key1" (hex) on stdin and prints the four output
// words of one block. In that engine the key is the seed, counter words 2-3
// are the subsequence and words 0-1 the offset in blocks.
#include <ATen/core/PhiloxRNGEngine.h>
#include <cstdio>

int main() {
  unsigned c0, c1, c2, c3, k0, k1;
  while (std::scanf("%x %x %x %x %x %x", &c0, &c1, &c2, &c3, &k0, &k1) == 6) {
    uint64_t seed = (uint64_t)k0 | ((uint64_t)k1 << 32);
    uint64_t subseq = (uint64_t)c2 | ((uint64_t)c3 << 32);
    uint64_t offset = (uint64_t)c0 | ((uint64_t)c1 << 32);
    at::Philox4_32 e(seed, subseq, 0);
    e.incr_n(offset);
    unsigned o0 = e(), o1 = e(), o2 = e(), o3 = e();
    std::printf("%08x %08x %08x %08x\n", o0, o1, o2, o3);
  }
  return 0;
}
