// Host-side check of the Q6_K K-slice split (q6k_slices.h) for every super-block count up to
// 4096: the slices tile [0, nsb) in order, their lengths differ by at most one with the longer
// ones first, q6_slice_ends marks exactly the last super-block of every non-empty slice, and
// the four SM sub-partitions (warps w, w+4, w+8, w+12) get loads that differ by at most one
// super-block -- seven each at nsb = 28 (K = 7168).
#include <cstdio>

#include "q6k_slices.h"

using dlmh::kQ6Slices;
using dlmh::q6_slice_begin;
using dlmh::q6_slice_ends;

int main() {
  for (int nsb = 1; nsb <= 4096; ++nsb) {
    if (q6_slice_begin(nsb, 0) != 0 || q6_slice_begin(nsb, kQ6Slices) != nsb)
      return printf("slices do not tile nsb=%d\n", nsb), 1;
    int prev_len = 1 << 30, nonempty = 0;
    int part[4] = {0, 0, 0, 0};
    for (int w = 0; w < kQ6Slices; ++w) {
      const int b = q6_slice_begin(nsb, w), e = q6_slice_begin(nsb, w + 1), len = e - b;
      if (len < 0 || len > prev_len) return printf("slice order nsb=%d w=%d\n", nsb, w), 1;
      if (len < nsb / kQ6Slices || len > nsb / kQ6Slices + 1) return printf("uneven nsb=%d w=%d\n", nsb, w), 1;
      prev_len = len;
      part[w % 4] += len;
      if (len > 0) {
        ++nonempty;
        for (int sb = b; sb < e; ++sb)
          if (q6_slice_ends(nsb, sb) != (sb == e - 1)) return printf("slice end nsb=%d sb=%d\n", nsb, sb), 1;
      }
    }
    if (nonempty != (nsb < kQ6Slices ? nsb : kQ6Slices)) return printf("non-empty count nsb=%d\n", nsb), 1;
    int lo = part[0], hi = part[0];
    for (int s = 1; s < 4; ++s) {
      lo = part[s] < lo ? part[s] : lo;
      hi = part[s] > hi ? part[s] : hi;
    }
    if (hi - lo > 1) return printf("sub-partition loads nsb=%d: %d..%d\n", nsb, lo, hi), 1;
    if (nsb == 28 && (lo != 7 || hi != 7)) return printf("nsb=28 not seven per sub-partition\n"), 1;
  }
  printf("ok 4096 super-block counts\n");
  return 0;
}
