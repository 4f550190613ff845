// Host-side mask -> tile work list.
//
// The Causal-rCM report (Appendix B, "Sparse custom-mask representation")
// streams only admissible query/key rectangles. Here the rectangles are the
// tiles of one global grid (query tiles of bm rows, key tiles of bn keys,
// anchored at token 0) and each tile is FULL (every in-range slot admitted),
// PARTIAL (some) or EMPTY (none, never visited). Keeping the global grid
// rather than restarting tiles at every range edge wastes fewer slots on
// ragged frame sizes (1560 = 12*128 + 24 tokens per frame).
#pragma once

#include <stdint.h>

#include <vector>

#include "../../include/jvp_attn.h"

namespace jvp {

// Returns JVP_OK or the error code for a bad descriptor / length.
int validate_mask(const jvp_mask_desc& m, int L);

// Admitted (query, key) pairs over all L rows.
int64_t count_pairs(const jvp_mask_desc& m, int L);

struct Schedule {
  int L = 0, bm = 0, bn = 0, n_qt = 0, n_kt = 0;
  int64_t n_full = 0, n_partial = 0, n_empty = 0;
  int64_t max_ktiles = 0;  // longest query tile, in key tiles
  // Per query tile, longest first: {qt, seg_begin, seg_count, n_ktiles}.
  std::vector<int32_t> qtiles;
  // Segments: {kt_begin, (kt_count << 1) | partial}.
  std::vector<int32_t> segs;
};

// Classifies one query tile's key tiles into out[0 .. n_kt).
void classify_qtile(const jvp_mask_desc& m, int L, int bm, int bn, int qt,
                    int8_t* out);

// Builds the full schedule. The mask must already be validated.
Schedule build_schedule(const jvp_mask_desc& m, int L, int bm, int bn);

// Key-tile-major work list for the backward's key/value pass: one entry per
// key tile of bk keys, {kt, seg_begin, seg_count, n_qtiles}, longest first,
// and segments of query tiles of bq rows {qt_begin, (count << 1) | partial}.
// A tile is FULL only if every (query, key) slot is admitted and neither
// its queries nor its keys reach past L (query rows past L must be masked
// here, since the pass reads per-query LSE and D values).
Schedule build_schedule_kv(const jvp_mask_desc& m, int L, int bq, int bk);

// Work list for chunk attention over a key/value cache: Lq query rows
// against the first Lk keys, all admitted, for BH (batch, head) pairs, on
// `grid` persistent CTAs taking items in list order. The items (bh, query
// tile of bq rows) of n_kt key tiles of bk keys each come first, whole and
// in (bh, query tile) order, as many as fill whole waves of the grid
// (concurrent CTAs then read the same key tiles of one head, which stay in
// L2). The r items left over are cut into about `grid` pieces in all (key
// ranges of near-equal length, at least 4 tiles where possible), listed
// piece-major so that concurrent CTAs again share key ranges. A piece of a
// cut item writes an fp32 partial into its own slot (the slots of an item
// are consecutive) for a combine step; a whole item writes the output
// itself. The last key tile is PARTIAL when Lk is not a multiple of bk.
struct CacheSchedule {
  int n_qt = 0, n_kt = 0, n_slots = 0;
  // Per piece, in list order: {qt, seg_begin, seg_count, n_ktiles}.
  std::vector<int32_t> entries;
  // Segments: {kt_begin, (kt_count << 1) | partial}.
  std::vector<int32_t> segs;
  // Per piece: {bh, partial slot, or -1 for a whole item}.
  std::vector<int32_t> meta;
  // Per cut item: {bh, qt, first slot, slot count}.
  std::vector<int32_t> splits;
};
CacheSchedule build_schedule_cache(int Lq, int Lk, int bq, int bk, int BH, int grid);

// The same work list as build_schedule (same entries, same order), written
// into caller-provided arrays without any heap allocation: entries of 4
// int32 to `qtiles`, segments of 2 int32 ({kt_begin, (count << 1) |
// partial}) to `segs`. Capacities are in int32 words. Returns false when a
// capacity is exceeded (*n_qt / *n_segs then hold what was counted so far).
// bm must be <= 256. The mask must already be validated.
bool build_schedule_into(const jvp_mask_desc& m, int L, int bm, int bn, int32_t* qtiles,
                         int64_t qtile_words, int32_t* segs, int64_t seg_words, int* n_qt,
                         int* n_segs);

}  // namespace jvp
