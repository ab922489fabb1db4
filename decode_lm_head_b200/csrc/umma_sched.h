// Hybrid stream-K schedule of the tensor-core GEMV (plain C++, shared by the kernels and
// by a host-side checker).  G CTAs; a unit is one pipeline stage (KC 128-byte chunks of one
// 128-row weight tile), spt units per tile.  CTA b first runs whole tiles [b wt, (b+1) wt);
// the last `rem` tiles (rem < G) are cut into units and CTA b also runs remainder units
// [b R / G, (b+1) R / G), R = rem * spt, which touch at most two tiles; their f32 sums go to
// partial slots 2b and 2b + 1 and a fixup pass adds them in unit (K) order.
#pragma once

#include <stdint.h>

#ifndef __CUDACC__
#define __host__
#define __device__
#endif

namespace dlmh {

struct Sched {
  int spt, wt, rem, G;
  __host__ __device__ int64_t r0(int b) const { return (int64_t)b * rem * spt / G; }
  // Remainder segment s (0 or 1) of CTA b: tile, unit range [u0, u1); false if absent.
  __host__ __device__ bool seg(int b, int s, int& tile, int& u0, int& u1) const {
    const int64_t a = r0(b), e = r0(b + 1);
    if (e <= a) return false;
    const int64_t tf = a / spt;
    if (s == 0) {
      tile = (int)tf;
      u0 = (int)(a - tf * spt);
      u1 = (int)(e - tf * spt < spt ? e - tf * spt : spt);
    } else {
      const int64_t next = (tf + 1) * spt;
      if (e <= next) return false;
      tile = (int)tf + 1;
      u0 = 0;
      u1 = (int)(e - next);
    }
    tile += wt * G;
    return true;
  }
  // Job j of CTA b: a whole tile (slot -1) or a remainder segment (partial slot 2b + s).
  __host__ __device__ bool job(int b, int j, int& tile, int& u0, int& u1, int& slot) const {
    if (j < wt) {
      tile = b * wt + j;
      u0 = 0;
      u1 = spt;
      slot = -1;
      return true;
    }
    const int s = j - wt;
    int t0, a0, e0;
    if (!seg(b, 0, t0, a0, e0)) return false;
    if (s == 0) {
      tile = t0, u0 = a0, u1 = e0, slot = 2 * b;
      return true;
    }
    if (s == 1 && seg(b, 1, tile, u0, u1)) {
      slot = 2 * b + 1;
      return true;
    }
    return false;
  }
  // The CTA whose remainder range holds remainder unit u (0 <= u < rem * spt).
  __host__ __device__ int owner(int64_t u) const {
    const int64_t R = (int64_t)rem * spt;
    int b = (int)(u * G / R);
    while (b > 0 && r0(b) > u) --b;
    while (b + 1 < G && r0(b + 1) <= u) ++b;
    return b;
  }
};

// Schedule of a weight of `ntiles` 128-row tiles, spt units each, on `sms` SMs.
inline Sched make_sched(int ntiles, int spt, int sms) {
  Sched s{spt, 0, 0, 0};
  if (ntiles >= sms) {
    s.G = sms;
    s.wt = ntiles / sms;
    s.rem = ntiles - s.wt * sms;
  } else {
    const int64_t units = (int64_t)ntiles * spt;
    s.G = units < sms ? (int)units : sms;
    s.rem = ntiles;
  }
  return s;
}

}  // namespace dlmh
