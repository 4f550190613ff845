"""The kernels' transposed mask (queries admitting a key) agrees with the
row form (keys admitted by a query) for every pair: compiled from the
library's own header with g++ and checked by brute force on the CPU."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "attention_jvp_continuous_b200", "csrc")

PROGRAM = r'''
#include <cstdio>
#include "mask_rows.cuh"
using namespace jvp;
int main() {
  long checked = 0;
  for (int mode = 0; mode < 4; ++mode)
    for (int T = 1; T <= 6; ++T)
      for (int F = 1; F <= 7; ++F)
        for (int ch = 1; ch <= 4; ++ch) {
          const int L = (mode == 3 ? 2 : 1) * T * F;
          for (int i = -1; i <= L; ++i)
            for (int j = -1; j <= L; ++j) {
              const bool a = key_ok(row_keys(mode, T, F, ch, L, i), j);
              const bool b = key_ok(key_queries(mode, T, F, ch, L, j), i);
              if (a != b) {
                std::printf("MISMATCH mode=%d T=%d F=%d ch=%d i=%d j=%d\n", mode, T, F, ch, i, j);
                return 1;
              }
              ++checked;
            }
        }
  std::printf("OK %ld\n", checked);
  return 0;
}
'''


def test_key_queries_is_transpose_of_row_keys():
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not available")
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "t.cpp")
        exe = os.path.join(d, "t")
        with open(src, "w") as f:
            f.write(PROGRAM)
        subprocess.run([gxx, "-std=c++17", "-O1", "-I", CSRC, src, "-o", exe], check=True)
        out = subprocess.run([exe], capture_output=True, text=True)
        assert out.returncode == 0, out.stdout
        assert out.stdout.startswith("OK")
