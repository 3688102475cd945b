"""Host checks of the attention kernels' work split (csrc/step_split.cuh).

The header is plain integer arithmetic marked __host__ __device__; this test
compiles it with the host C++ compiler and checks, over a grid of segment
counts, steps per segment and grid sizes, that every step of every segment is
dealt to exactly one CTA, that the CTAs' step counts differ by at most one,
that each piece stays inside its segment and that a CTA's run crosses at most
one segment boundary.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "lsh_bucketed_sparse_b200", "csrc", "step_split.cuh")

CHECKER = r"""
#define __host__
#define __device__
#define __forceinline__ inline
#include "step_split.cuh"
#include <cstdio>
#include <vector>
using namespace lsh;

// Returns the number of failed checks for one configuration.
static int check(long long segs, int steps, int n_h, int sms, long long* max_load) {
  int G;
  const StepSplit sp = make_step_split(segs, steps, sms, G);
  if (G < 1 || G > sms || G > sp.total) return 1;
  std::vector<int> seen(segs * steps, 0);
  long long mx = 0, mn = 1LL << 60;
  int bad = 0;
  for (int c = 0; c < G; ++c) {
    long long n = 0;
    for (int k = 0;; ++k) {
      if (k > 4 * (sp.full_rounds + 1) + 4) { ++bad; break; }  // no end marker
      Unit U;
      const int got = split_piece(sp, n_h, c, G, k, U);
      if (got == kPieceEnd) break;
      if (got == kPieceEmpty) continue;
      const long long seg = (long long)U.bh * n_h + U.r;
      if (U.r < 0 || U.r >= n_h || seg < 0 || seg >= segs || U.s0 < 0 || U.s0 >= U.s1 ||
          U.s1 > steps) { ++bad; break; }
      // a second piece of the same run starts its segment
      if ((k & 1) && U.s0 != 0) ++bad;
      for (int s = U.s0; s < U.s1; ++s) seen[seg * steps + s]++;
      n += U.s1 - U.s0;
    }
    mx = n > mx ? n : mx;
    mn = n < mn ? n : mn;
  }
  for (int x : seen) if (x != 1) { ++bad; break; }
  if (mx - mn > 1) ++bad;
  *max_load = mx;
  return bad;
}

int main() {
  int cases = 0, bad = 0;
  for (int n_h : {1, 2, 4, 8})
    for (long long bh : {1LL, 2LL, 3LL, 8LL, 32LL, 37LL})
      for (int steps : {1, 2, 3, 5, 8, 32, 96, 128, 333, 512})
        for (int sms : {1, 2, 7, 148}) {
          long long mx;
          const int b = check(bh * n_h, steps, n_h, sms, &mx);
          if (b) printf("fail: segs=%lld steps=%d n_h=%d sms=%d\n", bh * n_h, steps, n_h, sms);
          bad += b;
          ++cases;
        }
  // the long-text workload (64 segments of 512 steps) on 148 SMs: no CTA
  // walks more than one step above the mean of 221.4
  long long mx;
  bad += check(64, 512, 8, 148, &mx);
  if (mx != 222) { printf("long-text busiest CTA: %lld steps\n", mx); ++bad; }
  printf("cases %d bad %d\n", cases, bad);
  return bad ? 1 : 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="no host C++ compiler")
def test_step_split_covers_every_step_once_and_balances(tmp_path):
    src = tmp_path / "split_check.cpp"
    exe = tmp_path / "split_check"
    src.write_text(CHECKER)
    subprocess.run(["g++", "-O1", "-std=c++17", "-I", os.path.dirname(HEADER), str(src), "-o",
                    str(exe)], check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "bad 0" in r.stdout
