// Host-side mask -> tile work list (see schedule.h).
#include "schedule.h"

#include <algorithm>
#include <limits>

#include "mask_rows.cuh"

namespace jvp {

int validate_mask(const jvp_mask_desc& m, int L) {
  if (m.mode < JVP_MASK_DENSE || m.mode > JVP_MASK_TEACHER_FORCING)
    return JVP_ERR_INVALID_ARG;
  if (m.tokens_per_frame < 1 || m.n_frames < 1 || L < 1)
    return JVP_ERR_INVALID_ARG;
  if (m.chunk < 1 && m.mode != JVP_MASK_DENSE && m.mode != JVP_MASK_FRAME_CAUSAL)
    return JVP_ERR_INVALID_ARG;
  const int64_t ft = int64_t(m.tokens_per_frame) * m.n_frames;
  const int64_t want = m.mode == JVP_MASK_TEACHER_FORCING ? 2 * ft : ft;
  if (want > std::numeric_limits<int32_t>::max() / 2) return JVP_ERR_TOO_LARGE;
  if (want != L) return JVP_ERR_SHAPE_MISMATCH;
  return JVP_OK;
}

static inline int chunk_of(const jvp_mask_desc& m) {
  return m.chunk < 1 ? 1 : m.chunk;
}

int64_t count_pairs(const jvp_mask_desc& m, int L) {
  int64_t total = 0;
  for (int i = 0; i < L; ++i) {
    RowKeys r = row_keys(m.mode, m.tokens_per_frame, m.n_frames, chunk_of(m), L, i);
    if (r.b0 > r.a0) total += r.b0 - r.a0;
    if (r.b1 > r.a1) total += r.b1 - r.a1;
  }
  return total;
}

static inline int overlap(int a, int b, int lo, int hi) {
  const int x = std::max(a, lo), y = std::min(b, hi);
  return y > x ? y - x : 0;
}

void classify_qtile(const jvp_mask_desc& m, int L, int bm, int bn, int qt,
                    int8_t* out) {
  const int n_kt = (L + bn - 1) / bn;
  const int r0 = qt * bm;
  const int r1 = std::min(r0 + bm, L);
  // Distinct row classes of this query tile (consecutive rows mostly share
  // their admissible intervals; a tile spans few frames).
  std::vector<RowKeys> cls;
  for (int i = r0; i < r1; ++i) {
    RowKeys r = row_keys(m.mode, m.tokens_per_frame, m.n_frames, chunk_of(m), L, i);
    if (cls.empty() || cls.back().a0 != r.a0 || cls.back().b0 != r.b0 ||
        cls.back().a1 != r.a1 || cls.back().b1 != r.b1)
      cls.push_back(r);
  }
  for (int kt = 0; kt < n_kt; ++kt) {
    const int k0 = kt * bn;
    const int k1 = std::min(k0 + bn, L);
    const bool ragged = k0 + bn > L;
    bool all = !ragged, any = false;
    for (const RowKeys& r : cls) {
      const int ov = overlap(r.a0, r.b0, k0, k1) + overlap(r.a1, r.b1, k0, k1);
      if (ov != k1 - k0) all = false;
      if (ov > 0) any = true;
    }
    out[kt] = all ? JVP_TILE_FULL : (any ? JVP_TILE_PARTIAL : JVP_TILE_EMPTY);
  }
}

Schedule build_schedule(const jvp_mask_desc& m, int L, int bm, int bn) {
  Schedule s;
  s.L = L;
  s.bm = bm;
  s.bn = bn;
  s.n_qt = (L + bm - 1) / bm;
  s.n_kt = (L + bn - 1) / bn;
  std::vector<int8_t> row(s.n_kt);
  struct Entry {
    int qt, seg_begin, seg_count, n_kt;
  };
  std::vector<Entry> entries;
  entries.reserve(s.n_qt);
  for (int qt = 0; qt < s.n_qt; ++qt) {
    classify_qtile(m, L, bm, bn, qt, row.data());
    Entry e{qt, int(s.segs.size() / 2), 0, 0};
    int kt = 0;
    while (kt < s.n_kt) {
      const int8_t c = row[kt];
      if (c == JVP_TILE_EMPTY) {
        ++s.n_empty;
        ++kt;
        continue;
      }
      int k2 = kt;
      while (k2 < s.n_kt && row[k2] == c) ++k2;
      const int cnt = k2 - kt;
      s.segs.push_back(kt);
      s.segs.push_back((cnt << 1) | (c == JVP_TILE_PARTIAL ? 1 : 0));
      if (c == JVP_TILE_FULL) s.n_full += cnt; else s.n_partial += cnt;
      e.seg_count += 1;
      e.n_kt += cnt;
      kt = k2;
    }
    entries.push_back(e);
    s.max_ktiles = std::max<int64_t>(s.max_ktiles, e.n_kt);
  }
  // Longest-processing-time-first order for the persistent grid.
  std::stable_sort(entries.begin(), entries.end(),
                   [](const Entry& a, const Entry& b) { return a.n_kt > b.n_kt; });
  s.qtiles.reserve(entries.size() * 4);
  for (const Entry& e : entries) {
    s.qtiles.push_back(e.qt);
    s.qtiles.push_back(e.seg_begin);
    s.qtiles.push_back(e.seg_count);
    s.qtiles.push_back(e.n_kt);
  }
  return s;
}

}  // namespace jvp

namespace jvp {

bool build_schedule_into(const jvp_mask_desc& m, int L, int bm, int bn, int32_t* qtiles,
                         int64_t qtile_words, int32_t* segs, int64_t seg_words, int* n_qt,
                         int* n_segs) {
  const int nq = (L + bm - 1) / bm, nk = (L + bn - 1) / bn;
  *n_qt = nq;
  *n_segs = 0;
  if (bm > 256 || int64_t(nq) * 4 > qtile_words) return false;
  const int ch = chunk_of(m);
  RowKeys cls[256];
  int64_t ns = 0;
  for (int qt = 0; qt < nq; ++qt) {
    const int r0 = qt * bm, r1 = std::min(r0 + bm, L);
    int ncls = 0;
    for (int i = r0; i < r1; ++i) {
      const RowKeys r = row_keys(m.mode, m.tokens_per_frame, m.n_frames, ch, L, i);
      if (ncls == 0 || cls[ncls - 1].a0 != r.a0 || cls[ncls - 1].b0 != r.b0 ||
          cls[ncls - 1].a1 != r.a1 || cls[ncls - 1].b1 != r.b1)
        cls[ncls++] = r;
    }
    const int64_t seg_begin = ns;
    int seg_count = 0, total = 0;
    int run_start = -1, run_class = JVP_TILE_EMPTY;
    for (int kt = 0; kt <= nk; ++kt) {
      int c = JVP_TILE_EMPTY;
      if (kt < nk) {
        const int k0 = kt * bn, k1 = std::min(k0 + bn, L);
        bool all = k0 + bn <= L, any = false;
        for (int x = 0; x < ncls; ++x) {
          const int ov = overlap(cls[x].a0, cls[x].b0, k0, k1) +
                         overlap(cls[x].a1, cls[x].b1, k0, k1);
          if (ov != k1 - k0) all = false;
          if (ov > 0) any = true;
        }
        c = all ? JVP_TILE_FULL : (any ? JVP_TILE_PARTIAL : JVP_TILE_EMPTY);
      }
      if (c != run_class) {
        if (run_class != JVP_TILE_EMPTY) {
          if (2 * (ns + 1) > seg_words) {
            *n_segs = int(ns);
            return false;
          }
          const int cnt = kt - run_start;
          segs[2 * ns] = run_start;
          segs[2 * ns + 1] = (cnt << 1) | (run_class == JVP_TILE_PARTIAL ? 1 : 0);
          ++ns;
          ++seg_count;
          total += cnt;
        }
        run_start = kt;
        run_class = c;
      }
    }
    qtiles[4 * qt] = qt;
    qtiles[4 * qt + 1] = int32_t(seg_begin);
    qtiles[4 * qt + 2] = seg_count;
    qtiles[4 * qt + 3] = total;
  }
  *n_segs = int(ns);
  // Longest first, ties by query tile: the order build_schedule produces.
  struct E {
    int32_t qt, sb, sc, nk;
  };
  E* e = reinterpret_cast<E*>(qtiles);
  std::sort(e, e + nq, [](const E& a, const E& b) {
    return a.nk != b.nk ? a.nk > b.nk : a.qt < b.qt;
  });
  return true;
}

}  // namespace jvp

namespace jvp {

Schedule build_schedule_kv(const jvp_mask_desc& m, int L, int bq, int bk) {
  Schedule s;
  s.L = L;
  s.bm = bq;
  s.bn = bk;
  s.n_qt = (L + bq - 1) / bq;
  s.n_kt = (L + bk - 1) / bk;
  // Classes on the (bq x bk) grid, then read column by column.
  std::vector<int8_t> cls(size_t(s.n_qt) * s.n_kt);
  for (int qt = 0; qt < s.n_qt; ++qt) {
    int8_t* row = cls.data() + size_t(qt) * s.n_kt;
    classify_qtile(m, L, bq, bk, qt, row);
    if ((qt + 1) * bq > L)
      for (int kt = 0; kt < s.n_kt; ++kt)
        if (row[kt] == JVP_TILE_FULL) row[kt] = JVP_TILE_PARTIAL;
  }
  struct Entry {
    int kt, seg_begin, seg_count, n_qt;
  };
  std::vector<Entry> entries;
  entries.reserve(s.n_kt);
  for (int kt = 0; kt < s.n_kt; ++kt) {
    Entry e{kt, int(s.segs.size() / 2), 0, 0};
    int qt = 0;
    while (qt < s.n_qt) {
      const int8_t c = cls[size_t(qt) * s.n_kt + kt];
      if (c == JVP_TILE_EMPTY) {
        ++s.n_empty;
        ++qt;
        continue;
      }
      int q2 = qt;
      while (q2 < s.n_qt && cls[size_t(q2) * s.n_kt + kt] == c) ++q2;
      const int cnt = q2 - qt;
      s.segs.push_back(qt);
      s.segs.push_back((cnt << 1) | (c == JVP_TILE_PARTIAL ? 1 : 0));
      if (c == JVP_TILE_FULL) s.n_full += cnt; else s.n_partial += cnt;
      e.seg_count += 1;
      e.n_qt += cnt;
      qt = q2;
    }
    if (e.n_qt > 0) entries.push_back(e);  // a key no query admits has no work
    s.max_ktiles = std::max<int64_t>(s.max_ktiles, e.n_qt);
  }
  std::stable_sort(entries.begin(), entries.end(),
                   [](const Entry& a, const Entry& b) { return a.n_qt > b.n_qt; });
  for (const Entry& e : entries) {
    s.qtiles.push_back(e.kt);
    s.qtiles.push_back(e.seg_begin);
    s.qtiles.push_back(e.seg_count);
    s.qtiles.push_back(e.n_qt);
  }
  return s;
}

CacheSchedule build_schedule_cache(int Lq, int Lk, int bq, int bk, int BH, int grid) {
  CacheSchedule s;
  s.n_qt = (Lq + bq - 1) / bq;
  s.n_kt = (Lk + bk - 1) / bk;
  const bool ragged = Lk % bk != 0;
  const int64_t U = int64_t(BH) * s.n_qt;
  const int64_t n_whole = grid > 0 ? U / grid * grid : U;  // whole waves
  const int r = int(U - n_whole);                          // items left over
  // Appends one piece: key tiles [k0, k1) of item u.
  auto piece = [&](int64_t u, int k0, int k1, int slot) {
    const int seg_begin = int(s.segs.size() / 2);
    int nseg = 0;
    const int full_end = (ragged && k1 == s.n_kt) ? k1 - 1 : k1;
    if (full_end > k0) {
      s.segs.push_back(k0);
      s.segs.push_back((full_end - k0) << 1);
      ++nseg;
    }
    if (full_end < k1) {
      s.segs.push_back(full_end);
      s.segs.push_back((1 << 1) | 1);
      ++nseg;
    }
    s.entries.push_back(int32_t(u % s.n_qt));
    s.entries.push_back(seg_begin);
    s.entries.push_back(nseg);
    s.entries.push_back(k1 - k0);
    s.meta.push_back(int32_t(u / s.n_qt));
    s.meta.push_back(slot);
  };
  for (int64_t u = 0; u < n_whole; ++u) piece(u, 0, s.n_kt, -1);
  if (r == 0) return s;
  // About `grid` pieces over the r leftover items, at least 4 key tiles
  // each: item i gets p_i pieces, the first grid % r items one more.
  const int cap = std::max(1, s.n_kt / 4);
  std::vector<int> np(r), slot0(r, -1);
  int max_p = 0;
  for (int i = 0; i < r; ++i) {
    np[i] = std::min(cap, std::max(1, grid / r + (i < grid % r ? 1 : 0)));
    max_p = std::max(max_p, np[i]);
    if (np[i] > 1) {
      slot0[i] = s.n_slots;
      s.n_slots += np[i];
      const int64_t u = n_whole + i;
      s.splits.push_back(int32_t(u / s.n_qt));
      s.splits.push_back(int32_t(u % s.n_qt));
      s.splits.push_back(slot0[i]);
      s.splits.push_back(np[i]);
    }
  }
  // Piece-major order: concurrent CTAs take the same key range of the
  // leftover items, which share it in L2.
  for (int j = 0; j < max_p; ++j)
    for (int i = 0; i < r; ++i)
      if (j < np[i]) {
        const int k0 = int(int64_t(j) * s.n_kt / np[i]);
        const int k1 = int(int64_t(j + 1) * s.n_kt / np[i]);
        piece(n_whole + i, k0, k1, np[i] > 1 ? slot0[i] + j : -1);
      }
  return s;
}

}  // namespace jvp
