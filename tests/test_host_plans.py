"""Host-side tile plans of the Hessian kernel, checked on the CPU.

The plans are host code inside post_pruning_b200/csrc/hessian_tc.cu. The
test compiles that file into a small host program (nvcc cross-compiles the
device code; nothing runs on a GPU) whose main() walks the plans for every
width and checks:
  * band tiles: the super-block numbering is a bijection onto the 128 x 256
    tiles that meet the upper triangle (every width up to 32,768);
  * square tiles (widths with at most 148 squares of 128 x 128): at most one
    single-square tile, at most 148 CTAs, each tile's token splits tile
    [0, n) in order, and the reduction's blocks write every element of H
    exactly once, directly or as a mirror (widths up to 1024).
"""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "post_pruning_b200", "csrc")

HARNESS = r'''
#include "hessian_tc.cu"
#include <cstdio>
#include <vector>

namespace sgpt {
void count_launches(unsigned long long) {}   // the library's counter lives in api.cu
long long wait_limit_cycles() { return kDefaultWaitCycles; }   // the setting lives in api.cu too
}

int main() {
  using namespace sgpt;
  int bad = 0;
  for (int d = 32; d <= 32768; d += (d < 4096 ? 32 : 544)) {
    const int tm = (d + 127) / 128, tn = (d + 255) / 256;
    const long long T = band_start(tm, tn);
    for (int G : {4, 8, 12, 16, 24}) {
      std::vector<char> seen((size_t)tm * tn, 0);
      for (long long t = 0; t < T; ++t) {
        int ti = -1, tj = -1;
        grouped_tile(t, tm, tn, G, ti, tj);
        if (ti < 0 || ti >= tm || tj < 0 || tj >= tn || tj < ti / 2 || seen[(size_t)ti * tn + tj]++) {
          if (bad++ < 5) printf("band d=%d G=%d t=%lld -> (%d, %d)\n", d, G, t, ti, tj);
          break;
        }
      }
    }
  }
  for (int d = 32; d <= 2048; d += 32) {
    for (long long n : {1000LL, 262144LL}) {
      Plan p{};
      if (!plan_pairs(d, n, p)) {
        if (bad++ < 5) printf("no square plan d=%d\n", d);
        continue;
      }
      int singles = 0;
      if (p.pw.ncta > kMaxPairCtas) ++bad;
      for (int t = 0; t < p.pt.ntiles; ++t) {
        const PairTile& tl = p.pt.t[t];
        singles += tl.nsq == 1;
        long long at = 0;
        for (int s = 0; s < tl.ns; ++s) {
          const PairWork& w = p.pw.w[tl.first + s];
          if (w.a != tl.a || w.c1 != tl.c1 || w.c2 != tl.c2 || w.nsq != tl.nsq || w.t0 != at || w.t1 <= w.t0) ++bad;
          at = w.t1;
        }
        if (at != n) ++bad;
      }
      if (singles > 1) ++bad;
      if (n != 1000 || d > 1024) continue;
      // the reduction's blocks and the flush's element rules
      std::vector<int> cnt((size_t)d * d, 0);
      for (int t = 0; t < p.pt.ntiles; ++t) {
        const PairTile& tl = p.pt.t[t];
        for (int blk = 0; blk < 4 * tl.nsq; ++blk) {
          const int sq = blk >> 2, br = (blk >> 1) & 1, bc = blk & 1;
          const int a = tl.a, c = sq ? tl.c2 : tl.c1;
          const int bi0 = a * 128 + 64 * br, bj0 = c * 128 + 64 * bc;
          if (bi0 >= d || bj0 >= d || (c == a && br > bc)) continue;
          const int i0 = c >= a ? bi0 : bj0, j0 = c >= a ? bj0 : bi0;
          for (int r = 0; r < 64; ++r)
            for (int q = 0; q < 64; ++q) {
              const int i = i0 + r, j = j0 + q;
              if (i < d && j < d && j >= i) ++cnt[(size_t)i * d + j];
              if (i < d && j < d && i < j) ++cnt[(size_t)j * d + i];
            }
        }
      }
      for (size_t e = 0; e < cnt.size(); ++e)
        if (cnt[e] != 1) {
          if (bad++ < 5) printf("square d=%d element %zu written %d times\n", d, e, cnt[e]);
          break;
        }
    }
  }
  printf("bad=%d\n", bad);
  return bad != 0;
}
'''


def _nvcc():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return None


@pytest.mark.skipif(_nvcc() is None, reason="nvcc not found")
def test_hessian_tile_plans(tmp_path):
    src = tmp_path / "plans.cu"
    exe = tmp_path / "plans"
    src.write_text(HARNESS)
    r = subprocess.run([_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17",
                        "-I" + CSRC, "-I" + os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "bad=0" in r.stdout, r.stdout[-2000:]
