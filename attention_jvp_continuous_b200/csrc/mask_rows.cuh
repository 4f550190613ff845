// Admissible key intervals of one query row, for host (scheduler) and
// device (kernels) alike.
//
// Every query row of the four temporal masks admits at most two half-open
// key intervals [a0, b0) and [a1, b1) (b <= a means empty):
//   DENSE            [0, L)
//   FRAME_CAUSAL     [0, (frame(i)+1) * T)
//   CHUNK_CAUSAL     [0, min((chunk(i)+1) * chunk * T, F*T))
//   TEACHER_FORCING  clean i < F*T : [0, min((chunk(i)+1)*S, F*T))
//                    noisy i' = i - F*T, own chunk [c0, c1):
//                                  [0, c0) and [F*T + c0, F*T + c1)
// with S = chunk * T tokens per chunk (Causal-rCM report, Sec. 2.3 and
// Sec. 3.1.1 after Eq. 8; Appendix B "Sparse custom-mask representation").
// A row index outside [0, L) admits nothing.
#pragma once

#include <stdint.h>

#ifdef __CUDACC__
#define JVP_HD __host__ __device__ __forceinline__
#else
#define JVP_HD inline
#endif

namespace jvp {

struct RowKeys {
  int a0, b0, a1, b1;
};

// mode / T / F / chunk as in jvp_mask_desc; validated by the caller.
JVP_HD RowKeys row_keys(int mode, int T, int F, int chunk, int L, int i) {
  RowKeys r{0, 0, 0, 0};
  if (i < 0 || i >= L) return r;
  const int FT = T * F;
  if (mode == 0) {  // dense
    r.b0 = L;
    return r;
  }
  const int S = (mode == 1 ? 1 : chunk) * T;
  if (mode == 1 || mode == 2) {
    const int e = (i / S + 1) * S;
    r.b0 = e < FT ? e : FT;
    return r;
  }
  // teacher forcing
  if (i < FT) {
    const int e = (i / S + 1) * S;
    r.b0 = e < FT ? e : FT;
    return r;
  }
  const int ii = i - FT;
  const int c0 = (ii / S) * S;
  const int c1 = (c0 + S < FT) ? c0 + S : FT;
  r.b0 = c0;            // clean chunks strictly before (empty when c0 == 0)
  r.a1 = FT + c0;
  r.b1 = FT + c1;       // own noisy chunk
  return r;
}

JVP_HD bool key_ok(const RowKeys& r, int j) {
  return (j >= r.a0 && j < r.b0) || (j >= r.a1 && j < r.b1);
}

// The transpose: the query rows i whose admissible keys contain key j, again
// at most two half-open intervals (used by the backward's key/value pass):
//   DENSE            [0, L)
//   FRAME/CHUNK      [c0, F*T), c0 = first token of key j's chunk
//   TEACHER_FORCING  clean key j : clean queries [c0, F*T) and noisy queries
//                    of later chunks [F*T + c0 + S, 2 F*T)
//                    noisy key j' = j - F*T, own chunk [c0, c1): noisy
//                    queries [F*T + c0, F*T + c1)
// key_ok(row_keys(i), j) == key_ok(key_queries(j), i) for all i, j.
JVP_HD RowKeys key_queries(int mode, int T, int F, int chunk, int L, int j) {
  RowKeys r{0, 0, 0, 0};
  if (j < 0 || j >= L) return r;
  const int FT = T * F;
  if (mode == 0) {
    r.b0 = L;
    return r;
  }
  const int S = (mode == 1 ? 1 : chunk) * T;
  if (mode == 1 || mode == 2) {
    r.a0 = (j / S) * S;
    r.b0 = FT;
    return r;
  }
  if (j < FT) {
    const int c0 = (j / S) * S;
    r.a0 = c0;
    r.b0 = FT;
    const int n0 = c0 + S;
    if (n0 < FT) {
      r.a1 = FT + n0;
      r.b1 = 2 * FT;
    }
    return r;
  }
  const int jj = j - FT;
  const int c0 = (jj / S) * S;
  const int c1 = (c0 + S < FT) ? c0 + S : FT;
  r.a0 = FT + c0;
  r.b0 = FT + c1;
  return r;
}

}  // namespace jvp
