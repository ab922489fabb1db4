// Host-side check of the tensor-core GEMV's stream-K schedule (umma_sched.h): for many
// (SM count, tile count, units per tile) every (tile, unit) is run exactly once, a CTA has at
// most wt + 2 jobs, partial slots are unique and below 2G, and the fixup's walk over a
// remainder tile's contributors visits its units in order with the slots that hold them.
#include <algorithm>
#include <cstdio>
#include <set>
#include <vector>

#include "umma_sched.h"

using dlmh::Sched;

int main() {
  long cases = 0;
  for (int sms : {1, 2, 7, 132, 148})
    for (int ntiles = 1; ntiles <= 2000; ntiles += (ntiles < 40 ? 1 : 37))
      for (int spt : {1, 2, 3, 4, 5, 20, 56, 64}) {
        const Sched sc = dlmh::make_sched(ntiles, spt, sms);
        if (sc.G < 1 || sc.G > sms || sc.rem > sc.G) {
          printf("bad schedule sms=%d ntiles=%d spt=%d\n", sms, ntiles, spt);
          return 1;
        }
        std::vector<int> seen((size_t)ntiles * spt, 0), unit_slot((size_t)ntiles * spt, -2);
        std::set<int> slots;
        for (int b = 0; b < sc.G; ++b) {
          int nj = 0;
          for (int tile, u0, u1, slot; sc.job(b, nj, tile, u0, u1, slot); ++nj) {
            if (tile < 0 || tile >= ntiles || u0 < 0 || u1 > spt || u0 >= u1) return printf("bad job\n"), 1;
            if ((slot < 0) != (tile < sc.wt * sc.G)) return printf("whole/partial mismatch\n"), 1;
            if (slot >= 0 && (slot >= 2 * sc.G || !slots.insert(slot).second)) return printf("slot\n"), 1;
            for (int u = u0; u < u1; ++u) {
              seen[(size_t)tile * spt + u]++;
              unit_slot[(size_t)tile * spt + u] = slot;
            }
          }
          if (nj > sc.wt + 2) return printf("too many jobs\n"), 1;
        }
        for (int v : seen)
          if (v != 1) return printf("coverage sms=%d ntiles=%d spt=%d\n", sms, ntiles, spt), 1;
        for (int t = 0; t < sc.rem; ++t) {
          const long tu0 = (long)t * spt, tu1 = tu0 + spt;
          long covered = tu0;
          for (int bb = sc.owner(tu0); bb < sc.G && sc.r0(bb) < tu1; ++bb) {
            if (sc.r0(bb + 1) <= sc.r0(bb)) continue;
            const int slot = 2 * bb + (sc.r0(bb) / spt == t ? 0 : 1);
            const long a = std::max<long>(sc.r0(bb), tu0), e = std::min<long>(sc.r0(bb + 1), tu1);
            if (a != covered) return printf("gap in fixup walk\n"), 1;
            const int tile = sc.wt * sc.G + t;
            for (long u = a; u < e; ++u)
              if (unit_slot[(size_t)tile * spt + (u - tu0)] != slot) return printf("slot mismatch\n"), 1;
            covered = e;
          }
          if (covered != tu1) return printf("fixup walk incomplete\n"), 1;
        }
        ++cases;
      }
  printf("ok %ld\n", cases);
  return 0;
}
