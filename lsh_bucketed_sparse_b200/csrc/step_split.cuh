// How the persistent tensor-core attention kernels share out their steps.
//
// Step s of a (b*h, round) segment holds the queries of sorted slots
// [128 s, 128 s + 128) (two chunks of 64, or one of 128).  The steps of all
// segments are laid end to end, segment after segment (flat index
// f = seg * steps + s), and the grid of G CTAs walks them in rounds of G
// runs of `strip` steps: in full round j CTA c takes the run
// [j G strip + c strip, j G strip + (c + 1) strip); the R steps left after
// the last full round are dealt out as [base + c R / G, base + (c + 1) R / G).
// So each CTA gets the same number of steps give or take one, and at any time
// the grid works inside one window of G strip consecutive steps, a few heads'
// worth of rows, which keeps the gathers of keys and values in L2.  A run is
// at most `steps` long, so it crosses at most one segment boundary: each run
// is two pieces, the second often empty.  A piece that does not start its
// segment also loads the look-back block (the keys of chunk k - 1 for its
// first chunk k).
#pragma once

#include <algorithm>

namespace lsh {

struct StepSplit {
  long long total;  // steps of all segments
  int steps;        // steps per segment
  int strip;        // run length of a full round, 1 <= strip <= steps
  int full_rounds;  // total / (G * strip)
};

// A piece: steps [s0, s1) of segment (bh, r), s0 < s1.
struct Unit {
  int bh, r, s0, s1;
};

enum PieceKind { kPieceEnd = 0, kPieceRun = 1, kPieceEmpty = 2 };

// Piece k (run k / 2, half k % 2) of CTA c out of G: kPieceRun with U set,
// kPieceEmpty for an empty second half (go on with k + 1), kPieceEnd past the
// CTA's last piece.
__host__ __device__ __forceinline__ int split_piece(const StepSplit& sp, int n_h, int c, int G,
                                                    int k, Unit& U) {
  const int j = k >> 1;
  const long long round = (long long)G * sp.strip;
  long long a, b;
  if (j < sp.full_rounds) {
    a = j * round + (long long)c * sp.strip;
    b = a + sp.strip;
  } else if (j == sp.full_rounds) {
    const long long base = j * round, R = sp.total - base;
    a = base + c * R / G;
    b = base + (c + 1) * R / G;
  } else {
    return kPieceEnd;
  }
  const bool last = j == sp.full_rounds;
  if (a >= b) return last ? kPieceEnd : kPieceEmpty;
  const long long seg_end = (a / sp.steps + 1) * sp.steps;
  if (k & 1) {
    if (seg_end >= b) return last ? kPieceEnd : kPieceEmpty;
    a = seg_end;
  } else if (b > seg_end) {
    b = seg_end;
  }
  const long long seg = a / sp.steps;
  U.bh = (int)(seg / n_h);
  U.r = (int)(seg % n_h);
  U.s0 = (int)(a - seg * sp.steps);
  U.s1 = U.s0 + (int)(b - a);
  return kPieceRun;
}

// The split of `segs` segments of `steps` steps over at most `sms` CTAs:
// about six runs per CTA, each at least two steps; `grid` receives the CTA
// count (no more CTAs than steps).
inline StepSplit make_step_split(long long segs, int steps, int sms, int& grid) {
  StepSplit sp;
  sp.steps = steps;
  sp.total = segs * steps;
  grid = (int)std::min<long long>(sms, sp.total);
  long long strip = std::max<long long>(2, sp.total / ((long long)sms * 6));
  sp.strip = (int)std::min<long long>(strip, steps);
  sp.full_rounds = grid > 0 ? (int)(sp.total / ((long long)grid * sp.strip)) : 0;
  return sp;
}

}  // namespace lsh
