// Tensor-core masked attention JVP for B200 (sm_100a): tcgen05 + TMEM + TMA.
//
// Computes, per (batch*head, query tile of 128 rows), in one streaming pass
// over the admissible key tiles of 64 keys (Causal-rCM report, Appendix B,
// Eq. 42-45):
//   S   = Q K^T                         (d-deep MMA, fp32 in TMEM)
//   dS  = dQ K^T + Q dK^T               (one 2d-deep contraction in TMEM)
//   e   = 2^(c2 S - m)                  (c2 = scale * log2 e; m = row max)
//   l  += sum e,  g += sum e dS         (row state in registers)
//   A1  += e V                          (TMEM accumulator, 128 x 128 fp32)
//   A23 += (scale e dS) V + e dV        (second TMEM accumulator)
// finishing with O = A1/l, mu = scale g/l, dO = A23/l - mu O, and
// LSE = (m + log2 l) ln 2. All accumulators share one running max m and one
// rescale factor (Appendix B, after Eq. 45); the max is raised lazily, only
// when a row's new maximum exceeds it by more than 2^8, which is exact
// because the finish uses ratios only.
//
// Warp roles (384 threads, one CTA per SM, persistent over the work list):
//   warp 0       TMA producer: Q/dQ per query tile, K|dK and V|dV rings of 2
//   warp 1       TMEM owner; issues PV(t) and then S(t+2) (whole warp, one
//                elected lane)
//   warp 2       issues dS += dQ K^T(t) once S(t) has completed
//   warps 4..11  softmax/JVP state, P write-back to TMEM, epilogue: two
//                warpgroups, each taking 32 of a tile's 64 key columns of
//                every row (one row per thread), exchanging row maxima
// MMAs per 64-key tile: [S | Q dK^T] = Q [K ; dK]^T (N = 128), then
// dS += dQ K^T (N = 64), then [A1 | A23] += P [V | dV] (N = 256, P from
// TMEM), then A23 += (scale e dS) V (N = 128).
// TMEM (512 columns): S/dS double buffer at [0,256): buffer b holds S in
// columns [128b, 128b+64) and dS in [128b+64, 128b+128); the bf16 operands
// e and scale*e*dS overwrite the first 32 columns of S and dS of their
// buffer. A1 at [256,384), A23 at [384,512). MMA order per CTA is
// S(0) S(1) PV(0) S(2) PV(1) S(3) ..., so the softmax of tile t overlaps
// PV(t-1) and S(t+1) on the tensor pipe.
//
// Every mbarrier wait is bounded: on expiry the CTA records a timeout in the
// device error word, drains its own TMA copies and MMAs, frees TMEM and
// exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include <mutex>

#include "common.cuh"
#include "mask_rows.cuh"
#include "sm100_pipeline.cuh"
#include "sm100_ptx.cuh"

namespace jvp {
namespace sm100 {

using namespace jvp::ptx;

constexpr int BM = 128;  // query rows per tile = TMEM lanes
constexpr int BN = 64;   // keys per tile
constexpr int D = 128;   // head dim
constexpr int kThreads = 384;
constexpr float kTau = 8.0f;  // lazy rescale threshold, log2 units

// Shared memory map (byte offsets from a 1024-aligned base). Every operand
// tile is stored as two 128-byte-swizzled halves (head-dim columns 0-63 and
// 64-127), each rows x 128 B, exactly as the TMA box {64, rows} lands.
constexpr uint32_t kQHalf = BM * 128;          // 16 KB
constexpr uint32_t kKHalf = BN * 128;          //  8 KB
constexpr uint32_t SM_Q = 0;                   // Q  : 32 KB
constexpr uint32_t SM_DQ = 2 * kQHalf;         // dQ : 32 KB
constexpr uint32_t SM_K = 4 * kQHalf;          // K/dK ring: stage s at +32 KB*s
constexpr uint32_t SM_V = SM_K + 2 * 4 * kKHalf;  // V/dV ring
constexpr uint32_t kStageBytes = 4 * kKHalf;      // 32 KB: K|dK or V|dV
constexpr uint32_t SM_BAR = SM_V + 2 * kStageBytes;  // 196608
constexpr uint32_t kSmemBytes = SM_BAR + 512 + 4096 + 1024;  // + barriers, exchange, slack

// Barrier slots (8 bytes each) inside SM_BAR.
enum : uint32_t {
  B_QFULL = 0,
  B_QEMPTY = 1,
  B_KFULL = 2,    // 2 slots (S(t) complete releases K stage t&1: B_SFULL)
  B_VFULL = 4,    // 2
  B_PVD = 6,      // 2: PV(t) of buffer t&1 complete; also releases V stage t&1
  B_SFULL = 8,    // 2
  B_PFULL = 10,   // 2
  B_AFREE = 12,
  B_DRAIN = 13,
  B_XMAX = 14,    // 8 slots: [lane quarter][tile parity], softmax halves' max exchange
  B_XSUM = 22,    // 4 slots: [lane quarter], end-of-item l/g exchange
  B_IFULL = 26,   // 4 slots: work-item ring, published
  B_IEMPTY = 30,  // 4 slots: work-item ring, released
  B_DRAIN2 = 34,  // drain barrier of the second MMA warp
  B_SAFULL = 35,  // 2: S and Q dK^T of buffer t&1 complete (dQ K^T may still run)
  B_PDFULL = 39,  // 2: scale e dS of buffer t&1 written (B_PFULL: e written)
  kNumBars = 41
};
constexpr uint32_t SM_TMEM_SLOT = SM_BAR + 8 * kNumBars;  // u32: TMEM base
constexpr uint32_t SM_ABORT = SM_TMEM_SLOT + 4;           // u32: abort flag
constexpr uint32_t SM_RING = SM_ABORT + 4;                // 4 x i32: work-item ring
constexpr uint32_t SM_XCHG = SM_BAR + 512;                // 4 KB: softmax exchange
static_assert(SM_RING + 16 <= SM_XCHG, "barrier area overflow");

// TMEM columns.
constexpr uint32_t TM_A1 = 256;
constexpr uint32_t TM_A23 = 384;

constexpr uint32_t IDESC_S = ptx::idesc_bf16(BM, BN, false, false);       // 128 x 64
constexpr uint32_t IDESC_SK = ptx::idesc_bf16(BM, 2 * BN, false, false);  // 128 x 128
constexpr uint32_t IDESC_PV = ptx::idesc_bf16(BM, D, false, true);        // 128 x 128
constexpr uint32_t IDESC_PVV = ptx::idesc_bf16(BM, 2 * D, false, true);   // 128 x 256

struct Params {
  const int4* qtiles;  // {qt, seg_begin, seg_count, n_ktiles}
  const int2* segs;    // {kt_begin, (count << 1) | partial}
  int n_entries, n_segs, n_items, n_qt, n_kt;
  int L;
  jvp_mask_desc mask;
  float scale, c2;
  __nv_bfloat16* o;
  __nv_bfloat16* d_o;
  float* lse;
  unsigned* err;
  unsigned* item_ctr;  // zero at launch; CTAs take work items from it in list order
  unsigned long long wait_limit_ns;
  int stall_test;  // the MMA warp first waits on a phase that nothing completes
  // Scatter epilogue: 0 = rows go to o, d_o, lse ([B*H, L, d]); otherwise
  // row n of local head (b, h) goes to shard r = n / shard_len, row
  // n % shard_len, head h0 + h of [B, h_total, shard_len, d] in o_dst[r] etc.
  int n_shards, shard_len, h_local, h0, h_total;
  __nv_bfloat16* o_dst[kMaxShards];
  __nv_bfloat16* d_o_dst[kMaxShards];
  float* lse_dst[kMaxShards];
};

using pipe::wait_bar;
using pipe::drain_wait;
using pipe::ItemRing;
using pipe::Role;
using pipe::kProducer;
using pipe::kConsumerWarp;
using pipe::kRing;
using pipe::kRingReaders;
using Cursor = pipe::Cursor<Params>;

__global__ void __launch_bounds__(kThreads, 1)
jvp_attn_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_dq,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_dk,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_dv,
                      const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // Align the working base to 1024 B (required by the 128-byte swizzle atoms).
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  auto bar = [&](uint32_t slot) { return base + SM_BAR + 8u * slot; };
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(base_ptr + SM_ABORT);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    mbar_init(bar(B_QEMPTY), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_PVD + s), 1);
      mbar_init(bar(B_SFULL + s), 1);
      mbar_init(bar(B_SAFULL + s), 1);
      mbar_init(bar(B_PFULL + s), 2 * BM);
      mbar_init(bar(B_PDFULL + s), 2 * BM);
    }
    mbar_init(bar(B_AFREE), 2 * BM);
    mbar_init(bar(B_DRAIN), 1);
    mbar_init(bar(B_DRAIN2), 1);
    for (int i = 0; i < 8; ++i) mbar_init(bar(B_XMAX + i), 64);
    for (int i = 0; i < 4; ++i) mbar_init(bar(B_XSUM + i), 64);
    for (int i = 0; i < int(kRing); ++i) {
      mbar_init(bar(B_IFULL + i), 1);
      mbar_init(bar(B_IEMPTY + i), kRingReaders + 1);  // 3 MMA-warp cursors
    }
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tm_q);
    tma_prefetch_map(&tm_dq);
    tma_prefetch_map(&tm_k);
    tma_prefetch_map(&tm_dk);
    tma_prefetch_map(&tm_v);
    tma_prefetch_map(&tm_dv);
  }
  if (warp == 1) {
    tmem_alloc(base + SM_TMEM_SLOT, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(base_ptr + SM_TMEM_SLOT);
  const ItemRing ring{bar(B_IFULL), bar(B_IEMPTY),
                      reinterpret_cast<volatile int*>(base_ptr + SM_RING), abort_flag};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA ----
    if (lane == 0) {
      Cursor c;
      c.start(p, ring, kProducer);
      // How many times each full barrier was armed, for abort cleanup.
      // Stage s of a ring is armed by tiles t with t % 2 == s.
      uint32_t q_armed = 0, k_issued = 0, v_issued = 0;
      bool ok = true;
      while (c.valid && ok) {
        if (c.j == 0) {
          if (c.item_idx > 0)
            ok = wait_bar(bar(B_QEMPTY), (c.item_idx - 1) & 1, p, abort_flag);
          if (!ok) break;
          mbar_expect_tx(bar(B_QFULL), 4 * kQHalf);
          ++q_armed;
          const int y = c.qt * BM;
          tma_load_3d(base + SM_Q, &tm_q, bar(B_QFULL), 0, y, c.bh);
          tma_load_3d(base + SM_Q + kQHalf, &tm_q, bar(B_QFULL), 64, y, c.bh);
          tma_load_3d(base + SM_DQ, &tm_dq, bar(B_QFULL), 0, y, c.bh);
          tma_load_3d(base + SM_DQ + kQHalf, &tm_dq, bar(B_QFULL), 64, y, c.bh);
        }
        const uint32_t s = c.t & 1u, u = c.t >> 1;
        const int y = c.kt * BN;
        // Stage s is free once S(t - 2) is done: the S-ready barrier of that
        // buffer doubles as the K-stage release.
        if (c.t >= 2) ok = wait_bar(bar(B_SFULL + s), (u - 1) & 1u, p, abort_flag);
        if (!ok) break;
        mbar_expect_tx(bar(B_KFULL + s), kStageBytes);
        ++k_issued;
        // [K h0][dK h0][K h1][dK h1]: rows of K then dK are one 128-row
        // operand per head-dim half.
        const uint32_t ks = base + SM_K + s * kStageBytes;
        tma_load_3d(ks, &tm_k, bar(B_KFULL + s), 0, y, c.bh);
        tma_load_3d(ks + kKHalf, &tm_dk, bar(B_KFULL + s), 0, y, c.bh);
        tma_load_3d(ks + 2 * kKHalf, &tm_k, bar(B_KFULL + s), 64, y, c.bh);
        tma_load_3d(ks + 3 * kKHalf, &tm_dk, bar(B_KFULL + s), 64, y, c.bh);
        // V stage s is free once PV(t - 2) is done. PV(t - 4), the previous
        // phase of that barrier, was issued by warp 1 before S(t - 2), which
        // completed before dQ K^T(t - 2) was issued; that was waited for just
        // above, so the parity wait is unambiguous.
        if (c.t >= 2) ok = wait_bar(bar(B_PVD + s), (u - 1) & 1u, p, abort_flag);
        if (!ok) break;
        mbar_expect_tx(bar(B_VFULL + s), kStageBytes);
        ++v_issued;
        const uint32_t vs = base + SM_V + s * kStageBytes;
        tma_load_3d(vs, &tm_v, bar(B_VFULL + s), 0, y, c.bh);
        tma_load_3d(vs + kKHalf, &tm_v, bar(B_VFULL + s), 64, y, c.bh);
        tma_load_3d(vs + 2 * kKHalf, &tm_dv, bar(B_VFULL + s), 0, y, c.bh);
        tma_load_3d(vs + 3 * kKHalf, &tm_dv, bar(B_VFULL + s), 64, y, c.bh);
        c.next(p, ring, kProducer);
      }
      if (!ok || *abort_flag) {
        // Let copies already issued land before the CTA's smem is released.
        if (q_armed) drain_wait(bar(B_QFULL), (q_armed - 1) & 1u);
        for (uint32_t s = 0; s < 2; ++s) {
          const uint32_t nk = (k_issued + 1 - s) / 2, nv = (v_issued + 1 - s) / 2;
          if (nk) drain_wait(bar(B_KFULL + s), (nk - 1) & 1u);
          if (nv) drain_wait(bar(B_VFULL + s), (nv - 1) & 1u);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == 2) {
    // ----------------------------------------------------------- MMA ----
    // Issue is split over two warps, each running its loop as a whole warp
    // in uniform control flow with one elected lane issuing its MMAs and
    // commits. Warp 1 issues PV(t) ([A1 | A23] += P [V | dV], A23 += Pds V)
    // and then [S | Q dK^T](t+2) = Q [K ; dK]^T: S(t+2) overwrites the TMEM
    // buffer whose P PV(t) reads, and the MMAs of one thread run in issue
    // order. Warp 2 issues dS += dQ K^T(t) once the N=128 MMAs of tile t
    // have completed (their commit, which the softmax also waits for): MMAs
    // of different warps are ordered only through completions.
    {
      const bool w1 = warp == 1;
      bool ok = true;
      // Descriptors of the fixed shared-memory operands; an MMA's operand
      // is the base plus a compile-time byte offset >> 4 (the start-address
      // field stays below 2^14, so the add never carries out of it).
      const uint64_t q_desc = sdesc_sw128(base + SM_Q, 16, 1024);
      const uint64_t dq_desc = sdesc_sw128(base + SM_DQ, 16, 1024);
      const uint64_t k_desc = sdesc_sw128(base + SM_K, 16, 1024);       // stage 0
      const uint64_t v_desc = sdesc_sw128(base + SM_V, kKHalf, 1024);   // stage 0
      // Each wait first tests all of its barriers back to back (they are
      // normally complete already) and falls back to the bounded waits one
      // by one.
      // S(t): K|dK stage, and Q for a new item.
      auto wait_k = [&](const Cursor& c) -> bool {
        const uint32_t b = c.t & 1u, par = (c.t >> 1) & 1u;
        const bool need_q = c.j == 0;
        const bool r = mbar_test(bar(B_KFULL + b), par) &&
                       (!need_q || mbar_test(bar(B_QFULL), c.item_idx & 1));
        if (__all_sync(0xffffffffu, r)) return true;
        bool w = !need_q || wait_bar(bar(B_QFULL), c.item_idx & 1, p, abort_flag);
        w = w && wait_bar(bar(B_KFULL + b), par, p, abort_flag);
        return __all_sync(0xffffffffu, w);
      };
      // [S | Q dK^T] = Q [K ; dK]^T: one N=128 MMA per 16-wide k-step.
      auto issue_sa = [&](const Cursor& c) {
        const uint32_t b = c.t & 1u;
        const uint64_t kb = k_desc + b * (kStageBytes >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t oq = ((kk >> 2) * kQHalf + (kk & 3) * 32) >> 4;
          const uint32_t ob = ((kk >> 2) * (2 * kKHalf) + (kk & 3) * 32) >> 4;
          mma_ss_elect(tmem + b * 128u, q_desc + oq, kb + ob, IDESC_SK, kk > 0);
        }
        mma_commit_elect(bar(B_SAFULL + b));  // S ready: the softmax and warp 2 go on
      };
      if (w1) {
        Cursor cs, cp;  // S runs up to two tiles ahead of PV
        cs.start(p, ring, kConsumerWarp);
        cp.start(p, ring, kConsumerWarp);
        // Failure-detection test: wait on the drain barrier's first phase,
        // which nothing completes before this warp's own drain commit, so the
        // bounded wait runs out and the abort path below is taken.
        if (p.stall_test) ok = __all_sync(0xffffffffu, wait_bar(bar(B_DRAIN), 0u, p, abort_flag));
        for (int pre = 0; pre < 2 && ok && cs.valid; ++pre) {
          ok = wait_k(cs);
          if (!ok) break;
          tc_fence_after();
          issue_sa(cs);
          cs.next(p, ring, kConsumerWarp);
        }
        while (ok && cp.valid) {
          const uint32_t b = cp.t & 1u, par = (cp.t >> 1) & 1u;
          const bool need_a = cp.j == 0 && cp.item_idx > 0;
          const uint32_t pa = (cp.item_idx - 1) & 1;
          bool r = mbar_test(bar(B_PFULL + b), par);
          r = r && mbar_test(bar(B_VFULL + b), par);
          r = r && (!need_a || mbar_test(bar(B_AFREE), pa));
          if (!__all_sync(0xffffffffu, r)) {
            bool w = !need_a || wait_bar(bar(B_AFREE), pa, p, abort_flag);
            w = w && wait_bar(bar(B_PFULL + b), par, p, abort_flag);
            w = w && wait_bar(bar(B_VFULL + b), par, p, abort_flag);
            ok = __all_sync(0xffffffffu, w);
            if (!ok) break;
          }
          tc_fence_after();
          const uint64_t vb = v_desc + b * (kStageBytes >> 4);
          const uint32_t first = cp.j == 0 ? 0u : 1u;
          // [A1 | A23] += P [V | dV]: one N=256 MMA per 16-key step (A1 and
          // A23 are adjacent in TMEM; V h0, V h1, dV h0, dV h1 are 8 KB apart).
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks)
            mma_ts_elect(tmem + TM_A1, tmem + b * 128u + (ks >> 1) * 32u + (ks & 1) * 8u,
                         vb + ((ks * 2048) >> 4), IDESC_PVV, first | (ks > 0));
          // scale e dS is written after dS lands, once the softmax is done
          // with the exponentials.
          if (!__all_sync(0xffffffffu, mbar_test(bar(B_PDFULL + b), par))) {
            ok = __all_sync(0xffffffffu, wait_bar(bar(B_PDFULL + b), par, p, abort_flag));
            if (!ok) break;
          }
          tc_fence_after();
          // A23 += (scale e dS) V
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks)
            mma_ts_elect(tmem + TM_A23, tmem + b * 128u + 64u + (ks >> 1) * 32u + (ks & 1) * 8u,
                         vb + ((ks * 2048) >> 4), IDESC_PV, 1u);
          mma_commit_elect(bar(B_PVD + b));  // PV(t) done: V stage free, A1/A23 current
          cp.next(p, ring, kConsumerWarp);
          // S(t+2) follows PV(t) in this thread's order. (dQ K^T(t) has
          // completed too: the softmax waited for it before publishing the
          // scale e dS that PV(t) read.)
          if (cs.valid) {
            ok = wait_k(cs);
            if (!ok) break;
            tc_fence_after();
            issue_sa(cs);
            cs.next(p, ring, kConsumerWarp);
          }
        }
      } else {
        // dS = Q dK^T + dQ K^T: N=64 MMAs accumulate dQ K^T onto the N=128
        // result once it has completed. This warp waits for its own operands
        // (K stage, dQ) as well.
        Cursor c;
        c.start(p, ring, kConsumerWarp);
        while (ok && c.valid) {
          const uint32_t b = c.t & 1u, par = (c.t >> 1) & 1u;
          const bool need_q = c.j == 0;
          bool r = mbar_test(bar(B_SAFULL + b), par) && mbar_test(bar(B_KFULL + b), par) &&
                   (!need_q || mbar_test(bar(B_QFULL), c.item_idx & 1));
          if (!__all_sync(0xffffffffu, r)) {
            bool w = wait_bar(bar(B_SAFULL + b), par, p, abort_flag);
            w = w && wait_bar(bar(B_KFULL + b), par, p, abort_flag);
            w = w && (!need_q || wait_bar(bar(B_QFULL), c.item_idx & 1, p, abort_flag));
            ok = __all_sync(0xffffffffu, w);
            if (!ok) break;
          }
          tc_fence_after();
          const uint64_t kb = k_desc + b * (kStageBytes >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t oq = ((kk >> 2) * kQHalf + (kk & 3) * 32) >> 4;
            const uint32_t ob = ((kk >> 2) * (2 * kKHalf) + (kk & 3) * 32) >> 4;
            mma_ss_elect(tmem + b * 128u + 64u, dq_desc + oq, kb + ob, IDESC_S, 1u);
          }
          // dS ready; with the N=128 MMAs of tile t complete before these
          // were issued, this also releases K stage b (and, after the
          // item's last tile, Q and dQ).
          mma_commit_elect(bar(B_SFULL + b));
          if (c.j == c.n - 1) mma_commit_elect(bar(B_QEMPTY));
          c.next(p, ring, kConsumerWarp);
        }
      }
      if (__any_sync(0xffffffffu, !ok || *abort_flag)) {
        // Wait for every MMA this warp issued before TMEM is freed.
        const uint32_t db = bar(w1 ? B_DRAIN : B_DRAIN2);
        mma_commit_elect(db);
        drain_wait(db, 0);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ----------------------------------------------------- softmax / JVP ----
    // Two warpgroups share each row: warps 4-7 take columns [0, 32) of every
    // 64-key tile, warps 8-11 columns [32, 64). Warps 4+q and 8+q read the
    // same TMEM lane quarter q (rows 32q .. 32q+31) and exchange their
    // partial row maxima through shared memory every tile, so both halves
    // apply one running max. Their partial l and g are summed at the end.
    const int hw = (warp - 4) >> 2;                  // column half
    const int q4 = warp & 3;                         // TMEM lane quarter
    const int r = q4 * 32 + lane;                    // row within the tile
    const uint32_t tl = tmem + (uint32_t(q4 * 32) << 16);
    const int chunk = p.mask.chunk < 1 ? 1 : p.mask.chunk;
    float* const xmax = reinterpret_cast<float*>(base_ptr + SM_XCHG);   // [2][2][128]
    float* const xsum = xmax + 4 * BM;                                  // [2 (l,g)][2][128]
    Cursor c;
    c.start(p, ring, kConsumerWarp);
    float m_ref = -CUDART_INF_F, l = 0.f, g = 0.f;
    RowKeys rk{0, 0, 0, 0};
    int grow = 0;
    bool ok = true;
    while (c.valid) {
      if (c.j == 0) {
        grow = c.qt * BM + r;
        rk = row_keys(p.mask.mode, p.mask.tokens_per_frame, p.mask.n_frames, chunk, p.L, grow);
        m_ref = -CUDART_INF_F;
        l = 0.f;
        g = 0.f;
      }
      const uint32_t b = c.t & 1u;
      // S lands first (its own commit); dS = Q dK^T + dQ K^T completes while
      // the row max is taken and exchanged.
      ok = wait_bar(bar(B_SAFULL + b), (c.t >> 1) & 1u, p, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t sr[32], dr[32];
      tmem_ld32(tl + b * 128u + 32u * hw, sr);
      tmem_wait_ld();
      float s[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) s[i] = __uint_as_float(sr[i]);
      if (c.partial) {
        const int k0 = c.kt * BN + 32 * hw;
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (!key_ok(rk, k0 + i)) s[i] = -CUDART_INF_F;
      }
      // Partial row max as 8 independent chains, then the partner's half.
      float m8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) m8[i] = s[i];
#pragma unroll
      for (int i = 8; i < 32; ++i) m8[i & 7] = fmaxf(m8[i & 7], s[i]);
#pragma unroll
      for (int w2 = 4; w2 > 0; w2 >>= 1)
#pragma unroll
        for (int i = 0; i < w2; ++i) m8[i] = fmaxf(m8[i], m8[i + w2]);
      const uint32_t xp = b * 2u;  // exchange slot parity = tile parity
      xmax[(xp + hw) * BM + r] = m8[0];
      // Each half writes its P and scale e dS back over the S and dS
      // columns it read itself, so the exchange orders no TMEM accesses.
      mbar_arrive(bar(B_XMAX + q4 * 2 + b));
      ok = wait_bar(bar(B_XMAX + q4 * 2 + b), (c.t >> 1) & 1u, p, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      const float mxs = fmaxf(m8[0], xmax[(xp + (hw ^ 1)) * BM + r]) * p.c2;
      float alpha = 1.f;
      bool need = false;
      if (m_ref == -CUDART_INF_F) {
        m_ref = mxs;  // first admitted keys of this row: nothing to rescale yet
      } else if (mxs > m_ref + kTau) {
        alpha = ex2(m_ref - mxs);
        m_ref = mxs;
        need = true;
      }
      // Warps 4+q and 8+q hold the same rows and take the same decision.
      if (__any_sync(0xffffffffu, need)) {
        l *= alpha;
        g *= alpha;
        // A1/A23 hold PV(t-1); wait for it, then scale this quarter's rows:
        // the first warpgroup scales A1, the second A23.
        // (PV(t-3), the previous phase of that barrier, was issued by warp 1
        // before S(t), whose commit, covering all of that warp's earlier
        // MMAs, this warp has seen land.)
        ok = wait_bar(bar(B_PVD + ((c.t - 1) & 1u)), ((c.t - 1) >> 1) & 1u, p, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          const uint32_t col = (hw == 0 ? TM_A1 : TM_A23) + q * 32u;
          uint32_t a[32];
          tmem_ld32(tl + col, a);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) a[i] = __float_as_uint(__uint_as_float(a[i]) * alpha);
          tmem_st32(tl + col, a);
        }
        tmem_wait_st();
      }
      const float mref_use = m_ref == -CUDART_INF_F ? 0.f : m_ref;
      // First what needs only S: e = 2^(c2 s - m), l and the bf16 e that
      // P [V | dV] reads; then, once dS has landed (its N = 64 MMAs run
      // while the exponentials are computed), e dS, g and scale e dS for
      // A23 += (scale e dS) V. Pairs of columns in packed fp32 (f32x2)
      // arithmetic take one instruction per pair.
      const uint64_t c2v = f2pack(p.c2, p.c2), mv = f2pack(-mref_use, -mref_use);
      uint64_t ev[16];
      {
        uint64_t la = 0, lb = 0;  // 0 = two +0.0f
        uint32_t pp[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float x0, x1;
          f2unpack(fma2(f2pack(s[2 * i], s[2 * i + 1]), c2v, mv), x0, x1);
          const float e0 = ex2(x0), e1 = ex2(x1);
          ev[i] = f2pack(e0, e1);
          if (i & 1)
            lb = add2(lb, ev[i]);
          else
            la = add2(la, ev[i]);
          pp[i] = pack_bf16(e0, e1);
        }
        float u0, u1;
        f2unpack(add2(la, lb), u0, u1);
        l += u0 + u1;
        // bf16 e into S columns [32 hw, 32 hw + 16): a 16-key MMA step takes
        // its A operand from columns {0, 8, 32, 40}.
        tmem_st16(tl + b * 128u + 32u * hw, pp);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_PFULL + b));
      }
      ok = wait_bar(bar(B_SFULL + b), (c.t >> 1) & 1u, p, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      tmem_ld32(tl + b * 128u + 64u + 32u * hw, dr);
      tmem_wait_ld();
      {
        const uint64_t scv = f2pack(p.scale, p.scale);
        uint64_t ga = 0, gb = 0;
        uint32_t pd[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint64_t edv =
              mul2(ev[i], f2pack(__uint_as_float(dr[2 * i]), __uint_as_float(dr[2 * i + 1])));
          if (i & 1)
            gb = add2(gb, edv);
          else
            ga = add2(ga, edv);
          float q0, q1;
          f2unpack(mul2(edv, scv), q0, q1);
          pd[i] = pack_bf16(q0, q1);
        }
        float u0, u1;
        f2unpack(add2(ga, gb), u0, u1);
        g += u0 + u1;
        // scale e dS into dS columns [64 + 32 hw, 64 + 32 hw + 16).
        tmem_st16(tl + b * 128u + 64u + 32u * hw, pd);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_PDFULL + b));
      }

      if (c.j == c.n - 1) {
        // ------------------------------------------------------ epilogue --
        // PV(t) done. PV(t-2), the previous phase of this barrier, was issued
        // by warp 1 before S(t), whose commit (covering all of that warp's
        // earlier MMAs) this warp has seen land, so the parity wait is
        // unambiguous.
        ok = wait_bar(bar(B_PVD + (c.t & 1u)), (c.t >> 1) & 1u, p, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) break;
        // Row totals of l and g from both halves.
        xsum[hw * BM + r] = l;
        xsum[(2 + hw) * BM + r] = g;
        mbar_arrive(bar(B_XSUM + q4));
        ok = wait_bar(bar(B_XSUM + q4), c.item_idx & 1, p, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) break;
        const float lt = l + xsum[(hw ^ 1) * BM + r];
        const float gt = g + xsum[(2 + (hw ^ 1)) * BM + r];
        tc_fence_after();
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        const float mu = p.scale * gt * inv;
        const bool row_ok = grow < p.L;
        // Destination rows: this launch's [B*H, L, d] outputs, or (scatter
        // epilogue) the token-shard owner's buffers, possibly a peer GPU's
        // memory reached with plain stores over NVLink.
        __nv_bfloat16 *orow, *dorow;
        float* lrow;
        {
          const int n = row_ok ? grow : 0;
          if (p.n_shards == 0) {
            const size_t off = (size_t(c.bh) * p.L + n) * D;
            orow = p.o + off;
            dorow = p.d_o + off;
            lrow = p.lse + size_t(c.bh) * p.L + n;
          } else {
            const int r = n / p.shard_len, nr = n - r * p.shard_len;
            const int bb = c.bh / p.h_local, hh = c.bh - bb * p.h_local;
            const size_t row = (size_t(bb) * p.h_total + p.h0 + hh) * p.shard_len + nr;
            orow = p.o_dst[r] + row * D;
            dorow = p.d_o_dst[r] + row * D;
            lrow = p.lse_dst[r] + row;
          }
        }
        // This warpgroup writes head-dim columns [64 hw, 64 hw + 64).
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
          const uint32_t col = 64u * hw + 32u * cc;
          uint32_t a1[32], a23[32];
          tmem_ld32(tl + TM_A1 + col, a1);
          tmem_ld32(tl + TM_A23 + col, a23);
          tmem_wait_ld();
          uint32_t po[16], pdo[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float o0 = __uint_as_float(a1[2 * i]) * inv;
            const float o1 = __uint_as_float(a1[2 * i + 1]) * inv;
            const float d0 = __uint_as_float(a23[2 * i]) * inv - mu * o0;
            const float d1 = __uint_as_float(a23[2 * i + 1]) * inv - mu * o1;
            po[i] = pack_bf16(o0, o1);
            pdo[i] = pack_bf16(d0, d1);
          }
          if (row_ok) {
            uint4* go = reinterpret_cast<uint4*>(orow + col);
            uint4* gd = reinterpret_cast<uint4*>(dorow + col);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              go[i] = make_uint4(po[4 * i], po[4 * i + 1], po[4 * i + 2], po[4 * i + 3]);
              gd[i] = make_uint4(pdo[4 * i], pdo[4 * i + 1], pdo[4 * i + 2], pdo[4 * i + 3]);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(bar(B_AFREE));
        if (row_ok && hw == 0)
          *lrow =
              lt > 0.f ? (m_ref + log2f(lt)) * 0.69314718055994531f : -CUDART_INF_F;
      }
      c.next(p, ring, kConsumerWarp);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- host ----

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [BH, L, 128] bf16 viewed as a 3-D tensor (d innermost); box {64, rows, 1}.
static bool make_map(CUtensorMap* m, const void* ptr, int L, int BH, int rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(L), cuuint64_t(BH)};
  cuuint64_t strides[2] = {cuuint64_t(D) * 2, cuuint64_t(L) * D * 2};
  cuuint32_t box[3] = {64, cuuint32_t(rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace sm100

int launch_sm100(const LaunchArgs& a, const WorkList& w, int num_sms) {
  using namespace sm100;
  const int BH = a.B * a.H;
  CUtensorMap mq, mdq, mk, mdk, mv, mdv;
  if (!make_map(&mq, a.q, a.L, BH, BM) || !make_map(&mdq, a.dq, a.L, BH, BM) ||
      !make_map(&mk, a.k, a.L, BH, BN) || !make_map(&mdk, a.dk, a.L, BH, BN) ||
      !make_map(&mv, a.v, a.L, BH, BN) || !make_map(&mdv, a.dv, a.L, BH, BN))
    return JVP_ERR_LAUNCH_FAILED;
  Params p;
  p.qtiles = w.qtiles;
  p.segs = w.segs;
  p.n_entries = w.n_qtiles;
  p.n_segs = w.n_segs;
  const long long items = (long long)w.n_qtiles * BH;
  if (items > 0x7fffffffLL) return JVP_ERR_TOO_LARGE;
  p.n_items = int(items);
  p.n_qt = (a.L + BM - 1) / BM;
  p.n_kt = (a.L + BN - 1) / BN;
  p.L = a.L;
  p.mask = a.mask;
  p.scale = a.scale;
  p.c2 = a.scale * 1.4426950408889634f;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.d_o = static_cast<__nv_bfloat16*>(a.d_o);
  p.lse = a.lse;
  p.err = a.err;
  p.item_ctr = a.item_ctr;
  p.wait_limit_ns = a.wait_limit_ns;
  p.stall_test = a.stall_test ? 1 : 0;
  p.n_shards = a.n_shards;
  p.shard_len = a.n_shards > 0 ? a.L / a.n_shards : 0;
  p.h_local = a.H;
  p.h0 = a.h0;
  p.h_total = a.h_total;
  for (int r = 0; r < kMaxShards; ++r) {
    p.o_dst[r] = static_cast<__nv_bfloat16*>(a.o_dst[r]);
    p.d_o_dst[r] = static_cast<__nv_bfloat16*>(a.d_o_dst[r]);
    p.lse_dst[r] = a.lse_dst[r];
  }
  // The dynamic shared-memory opt-in is a per-device function attribute.
  static std::mutex attr_mu;
  static bool attr_done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return JVP_ERR_LAUNCH_FAILED;
  {
    std::lock_guard<std::mutex> lk(attr_mu);
    if (!attr_done[dev]) {
      if (cudaFuncSetAttribute(jvp_attn_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kSmemBytes) != cudaSuccess)
        return JVP_ERR_LAUNCH_FAILED;
      attr_done[dev] = true;
    }
  }
  const int grid = int(items < num_sms ? items : num_sms);
  if (!a.item_ctr || cudaMemsetAsync(a.item_ctr, 0, sizeof(unsigned), a.stream) != cudaSuccess)
    return JVP_ERR_LAUNCH_FAILED;
  jvp_attn_sm100_kernel<<<grid, kThreads, kSmemBytes, a.stream>>>(mq, mdq, mk, mdk, mv, mdv, p);
  return cudaGetLastError() == cudaSuccess ? JVP_OK : JVP_ERR_LAUNCH_FAILED;
}

}  // namespace jvp
