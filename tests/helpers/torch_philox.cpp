// Test helper: prints Philox4x32-10 words from torch's own CPU engine
// (ATen PhiloxRNGEngine), an implementation independent of the oracle.
// stdin: lines "seed subsequence offset n"; stdout: n words per line.
#include <ATen/core/PhiloxRNGEngine.h>
#include <cstdio>
#include <cinttypes>

int main() {
  unsigned long long seed, subseq, offset;
  int n;
  while (std::scanf("%llu %llu %llu %d", &seed, &subseq, &offset, &n) == 4) {
    at::philox_engine eng(seed, subseq, offset);
    for (int i = 0; i < n; ++i) std::printf(i ? " %u" : "%u", (unsigned)eng());
    std::printf("\n");
  }
  return 0;
}
