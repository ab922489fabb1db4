// Layout of the caller workspace of a tensor-core call (plain C++, shared by the library and
// by a host-side checker).  One workspace serves one stream's calls in order:
//
//   [0, 256)                     whole-tile queue: two ints, zero between launches
//   [codes_off, +codes_bytes)    W8A16 only: the two-term E4M3 codes of up to 128 rows
//                                (2 * roundup8(rows) rows of k bytes) and 128 float32 row
//                                multipliers 2^-e
//   [partial_off, +partial_bytes) stream-K partial sums: 2 slots per CTA, MMA-N columns of
//                                128 float32 weight rows each, when the schedule has a
//                                remainder
//
// Every region starts on a 256-byte boundary.  The sizes are a pure function of (split, tile
// count, k, rows of the widest pass, SM count): the schedule is the one the kernel runs.
#pragma once

#include <stdint.h>

#include "umma_sched.h"

namespace dlmh {

constexpr int kUmmaTileRows = 128;     // weight rows per tile (the MMA's M)
constexpr int kUmmaStageChunks = 4;    // 128-byte K chunks per schedule unit
constexpr int64_t kWsQueueBytes = 256;

inline int64_t ws_round256(int64_t v) { return (v + 255) / 256 * 256; }

// MMA N (B operand rows) of a pass over `rows` activation rows: W8A8 rows rounded up to 16;
// W8A16 the hi and lo terms, each rows rounded up to 8.
inline int umma_mma_n(bool split, int rows) { return split ? 2 * ((rows + 7) / 8 * 8) : (rows + 15) / 16 * 16; }

// From this MMA N up, the two CTAs of a party share each MMA on one TPC (M = 256, each CTA
// holding half of the activation box): the per-SM activation stream and its shared memory halve.
constexpr int kUmmaPairMinN = 128;
inline bool umma_pair_mode(int nb, int sms) { return nb >= kUmmaPairMinN && sms >= 2; }

// The schedule of every pass: parties of two CTAs (sms / 2 of them, at least one) over tile
// pairs, a pure function of the tile count, k and the SM count (never of the row count, so
// that both kernels give a tile the same K split at every row count).
inline Sched umma_schedule(int ntiles, int k, int sms) {
  const int spt = (k / 128 + kUmmaStageChunks - 1) / kUmmaStageChunks;
  return make_sched((ntiles + 1) / 2, spt, sms >= 2 ? sms / 2 : 1);
}

// Bytes of the stream-K partial sums of one pass (0 when every tile is whole): two slots per
// CTA of MMA-N columns of 128 float32 weight rows.
inline int64_t umma_partial_bytes(bool split, int ntiles, int k, int rows, int sms) {
  const Sched s = umma_schedule(ntiles, k, sms);
  if (s.rem <= 0) return 0;
  return (int64_t)2 * (2 * s.G) * umma_mma_n(split, rows) * kUmmaTileRows * (int64_t)sizeof(float);
}

// Bytes of the W8A16 code area of a pass over `rows` rows (codes + 128 row multipliers).
inline int64_t w8a16_code_bytes(int rows, int k) { return (int64_t)2 * ((rows + 7) / 8 * 8) * k + 128 * 4; }

struct WsLayout {
  int64_t codes_off, codes_bytes, partial_off, partial_bytes, total;
};

// Layout for calls of up to `rows` rows (the widest pass is min(rows, 128) rows; a narrower
// pass needs no more of any region).
inline WsLayout ws_layout(bool split, int ntiles, int k, int rows, int sms) {
  const int r = rows < 128 ? rows : 128;
  WsLayout L{};
  L.codes_off = kWsQueueBytes;
  L.codes_bytes = split ? w8a16_code_bytes(r, k) : 0;
  L.partial_off = L.codes_off + ws_round256(L.codes_bytes);
  L.partial_bytes = umma_partial_bytes(split, ntiles, k, r, sms);
  L.total = L.partial_off + L.partial_bytes;
  return L;
}

}  // namespace dlmh
