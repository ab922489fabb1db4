// Host-side check of the tensor-core GEMV's stream-K schedule (umma_sched.h): for many
// (SM count, tile count, units per tile) every (tile, unit) is run exactly once, a CTA has at
// most wt + 2 jobs, partial slots are unique and below 2G, and the fixup's walk over a
// remainder tile's contributors visits its units in order with the slots that hold them.
// Pair mode (two CTAs per party, tile pairs): every single tile's units are run once by the CTA
// of its half, the CTAs' partial slots are unique and inside the workspace size, and the pair
// fixup's walk finds them.
#include <algorithm>
#include <cstdio>
#include <set>
#include <vector>

#include "umma_sched.h"
#include "workspace_plan.h"

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
  // pair mode: party j = CTAs 2j + h; schedule tile T = single tiles 2T + h
  for (int sms : {2, 7, 132, 148})
    for (int ntiles = 1; ntiles <= 2000; ntiles += (ntiles < 40 ? 1 : 37))
      for (int spt : {1, 2, 5, 20, 40, 56}) {
        const int k = spt * dlmh::kUmmaStageChunks * 128;
        const Sched sc = dlmh::umma_schedule(ntiles, k, sms);
        const int ctas = 2 * sc.G;
        if (sc.G < 1 || ctas > sms || sc.spt != spt) return printf("bad pair schedule\n"), 1;
        const int64_t pbytes = dlmh::umma_partial_bytes(true, ntiles, k, 128, sms);
        const int64_t slot_bytes = (int64_t)256 * dlmh::kUmmaTileRows * 4;
        std::vector<int> seen((size_t)(ntiles + 1) * spt, 0), unit_slot((size_t)(ntiles + 1) * spt, -2);
        std::set<int> slots;
        for (int c = 0; c < ctas; ++c) {
          const int j = c / 2, h = c % 2;
          for (int nj = 0, t, u0, u1, slot; sc.job(j, nj, t, u0, u1, slot); ++nj) {
            const int tile = 2 * t + h;
            const int ps = slot < 0 ? -1 : 2 * c + (slot - 2 * j);
            if (tile > ntiles) return printf("pair tile past the phantom\n"), 1;
            if (ps >= 0 && (!slots.insert(ps).second || (int64_t)(ps + 1) * slot_bytes > pbytes))
              return printf("pair slot\n"), 1;
            for (int u = u0; u < u1; ++u) {
              seen[(size_t)tile * spt + u]++;
              unit_slot[(size_t)tile * spt + u] = ps;
            }
          }
        }
        for (int tile = 0; tile < ntiles; ++tile)
          for (int u = 0; u < spt; ++u)
            if (seen[(size_t)tile * spt + u] != 1) return printf("pair coverage\n"), 1;
        for (int t = 0; t < sc.rem; ++t)
          for (int h = 0; h < 2; ++h) {
            const long tu0 = (long)t * spt, tu1 = tu0 + spt;
            long covered = tu0;
            const int tile = 2 * (sc.wt * sc.G + t) + h;
            for (int bb = sc.owner(tu0); bb < sc.G && sc.r0(bb) < tu1; ++bb) {
              if (sc.r0(bb + 1) <= sc.r0(bb)) continue;
              const int slot = 2 * (2 * bb + h) + (sc.r0(bb) / spt == t ? 0 : 1);
              const long a = std::max<long>(sc.r0(bb), tu0), e = std::min<long>(sc.r0(bb + 1), tu1);
              if (a != covered) return printf("pair fixup gap\n"), 1;
              for (long u = a; u < e; ++u)
                if (unit_slot[(size_t)tile * spt + (u - tu0)] != slot) return printf("pair slot mismatch\n"), 1;
              covered = e;
            }
            if (covered != tu1) return printf("pair fixup incomplete\n"), 1;
          }
        ++cases;
      }
  printf("ok %ld\n", cases);
  return 0;
}
