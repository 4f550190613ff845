// Work distribution and bounded waits shared by the tensor-core kernels.
//
// A work item is (batch*head, outer tile) of a host-built work list: entries
// {outer tile, first segment, segment count, inner tiles} and segments
// {first inner tile, (count << 1) | partial}. CTAs take items dynamically
// from a global counter; a producer thread publishes each index into a
// 4-slot shared-memory ring that the other roles read. Every wait is
// bounded: on expiry it records a timeout in the device error word, raises
// the CTA's abort flag and returns false.
#pragma once

#include <stdint.h>

#include <type_traits>

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace jvp {
namespace pipe {

using namespace jvp::ptx;

// Slow path of wait_bar, kept out of line so that the hot loops stay small.
static __device__ __noinline__ bool wait_bar_slow(uint32_t bar, uint32_t parity,
                                           unsigned long long limit_ns, unsigned* err,
                                           volatile uint32_t* abort_flag) {
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try(bar, parity)) return true;
    // A try_wait may itself suspend for a while, so the limit is checked
    // from the first failed poll on.
    if ((it & 7u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > limit_ns) {
        atomicOr(err, kErrTimeout);
        *abort_flag = 1u;
        return false;
      }
    }
  }
}

// Bounded wait. Returns false (and raises the CTA abort flag) on timeout or
// when another role has already aborted.
template <class P>
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const P& p,
                                         volatile uint32_t* abort_flag) {
  // Most waits find the phase already complete: probe without suspending.
  if (mbar_test(bar, parity)) return true;
  return wait_bar_slow(bar, parity, p.wait_limit_ns, p.err, abort_flag);
}

// Work items reach the roles through a 4-slot ring in shared memory: the
// producer takes the next item index from the global counter (dynamic
// longest-first scheduling) and publishes it; every other role's cursor (a
// whole warp each: the MMA warps' and the softmax warps') reads it and
// releases the slot. Each kernel sets the slot's reader count.
enum Role { kProducer, kConsumerWarp };  // one producer thread; consumer warps
constexpr uint32_t kRing = 4;
constexpr uint32_t kRingReaders = 2 + 8;  // two MMA-warp cursors, eight softmax warps

struct ItemRing {
  uint32_t full_bar, empty_bar;  // first slot's mbarrier; slots are 8 B apart
  volatile int* slots;
  volatile uint32_t* abort_flag;
};

// Kernels whose parameters carry `piece_meta` ({bh, ...} per work item)
// list every item explicitly: item i is entry i of the work list, and its
// (batch*head) comes from piece_meta[i] instead of from the item index.
template <class P, class = void>
struct PieceMeta : std::false_type {};
template <class P>
struct PieceMeta<P, std::void_t<decltype(&P::piece_meta)>> : std::true_type {};

// Walks this CTA's (item, inner tile) sequence; every role runs its own copy.
// P provides: qtiles / segs (the work list), n_entries, n_segs, n_items,
// n_qt (outer tiles), n_kt (inner tiles), err, item_ctr, wait_limit_ns (and,
// for explicit item lists, piece_meta and n_bh).
template <class P>
struct Cursor {
  int item, item_idx, bh, qt;
  int seg, seg_end, kt, kt_end;
  int j, n;
  uint32_t t;  // ordinal of the tile among this CTA's tiles
  bool partial, valid;

  __device__ void load_seg(const P& p) {
    const int2 s = p.segs[seg];
    kt = s.x;
    kt_end = s.x + (s.y >> 1);
    partial = (s.y & 1) != 0;
    if (kt < 0 || kt_end > p.n_kt || kt_end <= kt) {
      atomicOr(p.err, kErrBounds);
      valid = false;
    }
  }
  // Index of this CTA's item number item_idx; false on timeout / abort.
  __device__ bool acquire(const P& p, const ItemRing& r, Role role) {
    const uint32_t slot = uint32_t(item_idx) % kRing, use = uint32_t(item_idx) / kRing;
    if (role == kProducer) {
      if (use > 0 && !wait_bar(r.empty_bar + 8 * slot, (use - 1) & 1u, p, r.abort_flag))
        return false;
      item = int(atomicAdd(p.item_ctr, 1u));
      r.slots[slot] = item;
      mbar_arrive(r.full_bar + 8 * slot);  // release: readers see the slot
      return true;
    }
    // A consumer is a whole warp: one arrive per warp releases the slot.
    const bool ok = __all_sync(0xffffffffu, wait_bar(r.full_bar + 8 * slot, use & 1u, p, r.abort_flag));
    if (!ok) return false;
    item = r.slots[slot];
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(r.empty_bar + 8 * slot);
    return true;
  }
  __device__ void load_item(const P& p, const ItemRing& r, Role role) {
    valid = acquire(p, r, role) && item < p.n_items;
    if (!valid) return;
    int e;
    if constexpr (PieceMeta<P>::value) {
      e = item;
      bh = p.piece_meta[item].x;
      if (bh < 0 || bh >= p.n_bh) {
        atomicOr(p.err, kErrBounds);
        valid = false;
        return;
      }
    } else {
      e = item % p.n_entries;
      bh = item / p.n_entries;
    }
    const int4 en = p.qtiles[e];
    qt = en.x;
    seg = en.y;
    seg_end = en.y + en.z;
    n = en.w;
    j = 0;
    if (qt < 0 || qt >= p.n_qt || seg < 0 || seg_end > p.n_segs || en.z < 1 || n < 1) {
      atomicOr(p.err, kErrBounds);
      valid = false;
      return;
    }
    load_seg(p);
  }
  __device__ void start(const P& p, const ItemRing& r, Role role) {
    item_idx = 0;
    t = 0;
    load_item(p, r, role);
  }
  __device__ void next(const P& p, const ItemRing& r, Role role) {
    ++t;
    ++j;
    if (++kt < kt_end) return;
    if (++seg < seg_end) {
      load_seg(p);
      return;
    }
    ++item_idx;
    load_item(p, r, role);
  }
};

// Short bounded wait used only while cleaning up after an abort.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try(bar, parity)) {
    if (globaltimer() - t0 > 100000000ull) return;  // 0.1 s
  }
}


}  // namespace pipe
}  // namespace jvp
