"""The work list of cache attention (build_schedule_cache): compiled from
the library's scheduler with g++ and checked on the CPU. Every (item, key
tile) pair appears in exactly one piece; the items that fill whole waves of
the grid come first, whole and in (bh, query tile) order; each leftover
item is cut into contiguous key ranges of near-equal length, at least four
tiles long where it has that many, about one piece per CTA in all, listed
piece-major; the pieces of a cut item carry consecutive slots that its
record lists, a whole item none; and only the tile holding key Lk - 1 is
partial, when Lk is not a multiple of the tile width."""
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
#define FAIL(msg) do { std::printf("BAD %s Lq=%d Lk=%d BH=%d G=%d\n", msg, Lq, Lk, BH, G); return 1; } while (0)
int main() {
  long checked = 0;
  // {Lq, Lk, BH, grid}
  const int cases[][4] = {{1560, 32760, 12, 148}, {4680, 32760, 12, 148}, {1, 1, 1, 148},
                          {128, 128, 1, 148}, {130, 300, 3, 7}, {7, 129, 2, 148},
                          {200, 65536, 5, 148}, {1, 255, 1, 3}, {3000, 1000, 40, 148},
                          {1560, 33000, 24, 132}, {1560, 32760, 1, 148}};
  for (const auto& cs : cases) {
    const int Lq = cs[0], Lk = cs[1], BH = cs[2], G = cs[3];
    const CacheSchedule s = build_schedule_cache(Lq, Lk, 128, 128, BH, G);
    const int nq = (Lq + 127) / 128, nk = (Lk + 127) / 128;
    const long U = long(BH) * nq, n_whole = U / G * G, r = U - n_whole;
    const int np = int(s.meta.size() / 2);
    if (int(s.entries.size()) != 4 * np) FAIL("pieces");
    std::vector<int> seen(size_t(U) * nk, 0), slot_used(size_t(s.n_slots), 0);
    std::vector<int> len_min(size_t(U), 1 << 30), len_max(size_t(U), 0), cnt(size_t(U), 0);
    long tail_pieces = 0;
    int prev_u = -1, prev_j_first = -1;
    for (int pc = 0; pc < np; ++pc) {
      const int qt = s.entries[4 * pc], sb = s.entries[4 * pc + 1];
      const int sc = s.entries[4 * pc + 2], n = s.entries[4 * pc + 3];
      const int bh = s.meta[2 * pc], slot = s.meta[2 * pc + 1];
      if (bh < 0 || bh >= BH || qt < 0 || qt >= nq) FAIL("item");
      const long u = long(bh) * nq + qt;
      int tot = 0, prev_end = -1, k_first = -1;
      for (int g = sb; g < sb + sc; ++g) {
        const int k0 = s.segs[2 * g], c = s.segs[2 * g + 1] >> 1, part = s.segs[2 * g + 1] & 1;
        if (prev_end >= 0 && k0 != prev_end) FAIL("gap");
        if (k_first < 0) k_first = k0;
        prev_end = k0 + c;
        for (int kt = k0; kt < k0 + c; ++kt) {
          const bool should_part = (Lk % 128 != 0) && kt == nk - 1;
          if (part != (should_part ? 1 : 0)) FAIL("partial flag");
          if (kt < 0 || kt >= nk) FAIL("range");
          seen[size_t(u) * nk + kt] += 1;
          ++checked;
        }
        tot += c;
      }
      if (tot != n || n < 1) FAIL("count");
      const bool whole = k_first == 0 && prev_end == nk;
      if (whole != (slot < 0)) FAIL("slot of a whole item");
      if (pc < n_whole) {
        if (u != pc || !whole) FAIL("whole waves first, in order");
      } else {
        if (u < n_whole) FAIL("leftover item");
        ++tail_pieces;
        // piece-major: the key range starts never move backwards
        if (prev_j_first > k_first && u <= prev_u) FAIL("piece-major order");
        prev_u = int(u);
        prev_j_first = k_first;
      }
      if (slot >= 0 && (slot >= s.n_slots || slot_used[size_t(slot)]++)) FAIL("slot reuse");
      len_min[size_t(u)] = n < len_min[size_t(u)] ? n : len_min[size_t(u)];
      len_max[size_t(u)] = n > len_max[size_t(u)] ? n : len_max[size_t(u)];
      cnt[size_t(u)] += 1;
    }
    for (int v : seen) if (v != 1) FAIL("cover");
    for (long u = n_whole; u < U; ++u) {
      if (len_max[size_t(u)] - len_min[size_t(u)] > 1) FAIL("piece balance");
      if (cnt[size_t(u)] > 1 && nk >= 4 && len_min[size_t(u)] < 4) FAIL("short piece");
    }
    if (r > 0) {
      long cap_total = r * (nk / 4 > 1 ? nk / 4 : 1);
      long want = G < cap_total ? G : cap_total;
      if (tail_pieces < (want > r ? want : r) || tail_pieces > (G > r ? G : r)) FAIL("tail pieces");
    }
    std::vector<int> listed(size_t(s.n_slots), 0);
    for (size_t i = 0; i + 3 < s.splits.size(); i += 4) {
      const int bh = s.splits[i], qt = s.splits[i + 1], s0 = s.splits[i + 2], ns = s.splits[i + 3];
      if (ns < 2 || s0 < 0 || s0 + ns > s.n_slots) FAIL("split record");
      for (int k = s0; k < s0 + ns; ++k) listed[size_t(k)] += 1;
      for (int pc = 0; pc < np; ++pc) {
        const int slot = s.meta[2 * pc + 1];
        if (slot >= s0 && slot < s0 + ns &&
            (s.meta[2 * pc] != bh || s.entries[4 * pc] != qt)) FAIL("split item");
      }
    }
    for (int v : listed) if (v != 1) FAIL("slots listed");
  }
  std::printf("OK %ld\n", checked);
  return 0;
}
'''


def test_cache_schedule():
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
