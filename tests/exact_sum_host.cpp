// Host driver for the exact +-1 Hadamard sum of the encoder (test only):
// reads "b o w0 w1 ... w(b-1)" lines (BF16 bit patterns in hex) from stdin and
// prints RN64 of sum_l (-1)^popcount(o & l) w_l as a hex float per line.
#include <cstdio>
#include <cstdint>
#include <vector>

#include "exact_sum.cuh"

int main() {
  int b, o;
  while (std::scanf("%d %d", &b, &o) == 2) {
    std::vector<uint16_t> w(b);
    for (int l = 0; l < b; ++l) {
      unsigned v;
      if (std::scanf("%x", &v) != 1) return 1;
      w[l] = (uint16_t)v;
    }
    std::printf("%a\n", dvssq::exact_pm_sum(w.data(), b, o));
  }
  return 0;
}
