"""The split work list of cache attention (build_schedule_dense): compiled
from the library's scheduler with g++ and checked on the CPU. Every
(query tile, key tile) pair appears exactly once, each split is a
contiguous key range of near-equal length, and only the tile holding key
Lk - 1 is partial, when Lk is not a multiple of the tile width."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "attention_jvp_continuous_b200", "csrc")

PROGRAM = r'''
#include <cstdio>
#include <vector>
#include "schedule.h"
using namespace jvp;
int main() {
  long checked = 0;
  const int cases[][3] = {{1, 1, 1}, {128, 128, 1}, {1560, 32760, 8}, {1560, 32760, 16},
                          {130, 300, 3}, {4680, 1000, 1}, {7, 129, 2}, {200, 65536, 64},
                          {1, 255, 2}};
  for (const auto& cs : cases) {
    const int Lq = cs[0], Lk = cs[1], S = cs[2];
    const Schedule s = build_schedule_dense(Lq, Lk, 128, 128, S);
    const int nq = (Lq + 127) / 128, nk = (Lk + 127) / 128;
    if (int(s.qtiles.size()) != 4 * nq * S) { std::printf("BAD entries %d %d\n", Lq, Lk); return 1; }
    std::vector<int> seen(size_t(nq) * nk, 0);
    int min_len = 1 << 30, max_len = 0;
    for (int e = 0; e < nq * S; ++e) {
      const int qt = s.qtiles[4 * e], sb = s.qtiles[4 * e + 1], sc = s.qtiles[4 * e + 2];
      const int n = s.qtiles[4 * e + 3];
      if (qt != e % nq) { std::printf("BAD order\n"); return 1; }
      int tot = 0, prev_end = -1;
      for (int g = sb; g < sb + sc; ++g) {
        const int k0 = s.segs[2 * g], cnt = s.segs[2 * g + 1] >> 1, part = s.segs[2 * g + 1] & 1;
        if (prev_end >= 0 && k0 != prev_end) { std::printf("BAD gap\n"); return 1; }
        prev_end = k0 + cnt;
        for (int kt = k0; kt < k0 + cnt; ++kt) {
          const bool should_part = (Lk % 128 != 0) && kt == nk - 1;
          if (part != (should_part ? 1 : 0)) { std::printf("BAD partial flag\n"); return 1; }
          if (kt < 0 || kt >= nk) { std::printf("BAD range\n"); return 1; }
          seen[size_t(qt) * nk + kt] += 1;
          ++checked;
        }
        tot += cnt;
      }
      if (tot != n) { std::printf("BAD count\n"); return 1; }
      min_len = n < min_len ? n : min_len;
      max_len = n > max_len ? n : max_len;
    }
    for (int v : seen) if (v != 1) { std::printf("BAD cover %d %d\n", Lq, Lk); return 1; }
    if (max_len - min_len > 1) { std::printf("BAD balance\n"); return 1; }
  }
  std::printf("OK %ld\n", checked);
  return 0;
}
'''


def test_dense_split_schedule():
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not available")
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "t.cpp")
        exe = os.path.join(d, "t")
        with open(src, "w") as f:
            f.write(PROGRAM)
        subprocess.run([gxx, "-std=c++17", "-O1", "-I", CSRC, src,
                        os.path.join(CSRC, "schedule.cpp"), "-o", exe], check=True)
        out = subprocess.run([exe], capture_output=True, text=True)
        assert out.returncode == 0, out.stdout
        assert out.stdout.startswith("OK")
