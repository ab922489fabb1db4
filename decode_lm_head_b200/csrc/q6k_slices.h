// K-slices of the Q6_K kernels (plain C++, shared by the kernels and by a host-side checker).
// The nsb super-blocks of a weight row are split into kQ6Slices slices as evenly as possible,
// the longer slices first.  The 8-row kernels run slice w on warp w; every Q6_K kernel
// accumulates each slice alone from 0 and adds the slices in order, so the split is part of
// the arithmetic they share.  At nsb = 28 (K = 7168) slices 0..11 hold two super-blocks and
// 12..15 one: each SM sub-partition (warps w, w+4, w+8, w+12) gets seven.
#pragma once

#ifdef __CUDACC__
#define DLMH_Q6_HD __host__ __device__ __forceinline__
#else
#define DLMH_Q6_HD inline
#endif

namespace dlmh {

constexpr int kQ6Slices = 16;

// First super-block of slice w (0 <= w <= kQ6Slices; slice w is [begin(w), begin(w + 1))).
DLMH_Q6_HD int q6_slice_begin(int nsb, int w) {
  const int q = nsb / kQ6Slices, r = nsb % kQ6Slices;
  return w * q + (w < r ? w : r);
}

// Whether a slice ends with super-block sb: the r slices of q + 1 end at multiples of q + 1,
// the others every q super-blocks after them (q = 0: every super-block ends one).
DLMH_Q6_HD bool q6_slice_ends(int nsb, int sb) {
  const int q = nsb / kQ6Slices, r = nsb % kQ6Slices;
  const int e = sb + 1, long_end = r * (q + 1);
  return e <= long_end ? e % (q + 1) == 0 : (e - long_end) % q == 0;
}

}  // namespace dlmh
