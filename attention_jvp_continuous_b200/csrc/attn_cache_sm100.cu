// Chunk attention over a key/value cache for B200 (sm_100a): the read-only
// forward of causal rollout (Causal-rCM report, Sec. 3.2.1 "KV Cache"): the
// Lq queries of the current chunk attend to the first Lk rows of the cache
// (the committed prefix the chunk needs, followed by the chunk's own keys
// at their cache position). O = softmax(c Q K^T) V and LSE per query row.
//
// One persistent tcgen05 kernel, one CTA per SM, 384 threads:
//   warp 0       TMA: Q once per item, K (3 stages) and V (2 stages) of 128
//                keys; the cache is read through tensor maps whose row
//                extent is Lk, so rows past the exposed prefix are zero-filled
//   warp 1       TMEM owner; issues S = Q K^T (N = 128) into a double
//                buffer
//   warp 2       issues O += P V (N = 128, P from TMEM); S(t+2) is issued
//                once PV(t) has completed (MMAs of different warps are
//                ordered only through completions)
//   warps 4-11   softmax: two warpgroups, each 64 of a tile's 128 keys of
//                every row with its own running max and its own O
//                accumulator (lazy rescale only when its row max grows by
//                more than 2^8); the epilogue merges the two halves
// Work items are (batch*head, 128-query tile) pairs over all key tiles, as
// many as fill whole waves of the grid, in head-major order (the CTAs
// running at once read the same key tiles of a head, served from L2); the
// items left over are cut into about one key-range piece per SM, listed
// piece-major so that concurrent CTAs again share key ranges. A whole item
// writes O and LSE itself; a piece writes an unnormalised fp32 partial (O,
// running max, sum) into its own slot, and a second kernel combines the
// pieces of each cut item. CTAs take items dynamically, in list order.
//
// TMEM: S buffer b at [128 b, 128 b + 128), the bf16 P of each key half
// packed over the start of that half's S columns; O_a at [256, 384) and O_b
// at [384, 512). Every mbarrier wait is bounded as in the JVP kernel.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include <mutex>

#include "common.cuh"
#include "sm100_pipeline.cuh"
#include "sm100_ptx.cuh"

namespace jvp {
namespace cache {

using namespace jvp::ptx;
using pipe::drain_wait;
using pipe::ItemRing;
using pipe::kConsumerWarp;
using pipe::kProducer;
using pipe::kRing;
using pipe::kRingReaders;
using pipe::wait_bar;

constexpr int BM = 128;  // query rows per tile = TMEM lanes
constexpr int BN = 128;  // keys per tile
constexpr int D = 128;
constexpr int kThreads = 384;
constexpr float kTau = 8.0f;  // lazy rescale threshold, log2 units
constexpr uint32_t NK = 3, NV = 2;

constexpr uint32_t kHalf = 128 * 128;   // 16 KB: 128 rows x 64 head-dim columns
constexpr uint32_t kStage = 2 * kHalf;  // 32 KB: one 128-row operand
constexpr uint32_t SM_Q = 0;
constexpr uint32_t SM_K = kStage;
constexpr uint32_t SM_V = SM_K + NK * kStage;
constexpr uint32_t SM_BAR = SM_V + NV * kStage;  // 192 KB
constexpr uint32_t SM_XCHG = SM_BAR + 512;       // softmax exchange
constexpr uint32_t kSmemBytes = SM_XCHG + 4096 + 1024;

enum : uint32_t {
  B_QFULL = 0,
  B_QEMPTY = 1,
  B_KFULL = 2,    // 3
  B_KEMPTY = 5,   // 3
  B_VFULL = 8,    // 2
  B_VEMPTY = 10,  // 2
  B_SFULL = 12,   // 2
  B_PFULL = 14,   // 2
  B_PVD = 16,     // 2: PV MMAs of the buffer's latest tile complete
  B_AFREE = 18,   // O read by the epilogue
  B_DRAIN = 19,
  B_XSUM = 20,    // 4: [lane quarter], end-of-item merge of the halves
  B_IFULL = 24,   // 4
  B_IEMPTY = 28,  // 4
  B_DRAIN2 = 34,  // drain barrier of the PV-issuing warp
  kNumBars = 35
};
constexpr uint32_t SM_TMEM_SLOT = SM_BAR + 8 * kNumBars;
constexpr uint32_t SM_ABORT = SM_TMEM_SLOT + 4;
constexpr uint32_t SM_RING = SM_ABORT + 4;
static_assert(SM_RING + 16 <= SM_XCHG, "barrier area overflow");
static_assert(kSmemBytes <= 232448, "shared memory over the per-block limit");

// Two O accumulators, one per key half of every tile (each softmax
// warpgroup keeps its own running max for its half; the halves are merged
// once per item in the epilogue).
constexpr uint32_t TM_O = 256;  // O_a [256, 384) for keys [0, 64), O_b [384, 512) for [64, 128)
constexpr uint32_t IDESC_S = ptx::idesc_bf16(BM, BN, false, false);  // 128 x 128, K-major B
constexpr uint32_t IDESC_PV = ptx::idesc_bf16(BM, D, false, true);   // 128 x 128, MN-major B

// 2^x for a pair on the FMA pipe, for the share of the exponentials that the
// MUFU unit (16 per cycle per SM, as many per tile as the tensor pipe has
// cycles of work here) would otherwise serialise. Cody-Waite range
// reduction: x = n + f with n = round(x), taken from the low bits of
// x + 1.5 * 2^23, and |f| <= 1/2; 2^f from a cubic whose coefficients were
// fitted here by iteratively reweighted least squares on [-1/2, 1/2]
// (relative error below 8e-5 in fp32, well inside the bf16 rounding of P);
// 2^n assembled in the exponent field. x is clamped at -127 first, where
// 2^n is exactly 0, so masked entries (x = -inf) give 0. Range: x <= 127.
__device__ __forceinline__ uint64_t ex2_fma2(float x0, float x1) {
  constexpr float kShift = 12582912.f;  // 1.5 * 2^23: ulp 1, round to nearest
  const uint64_t xv = f2pack(fmaxf(x0, -127.f), fmaxf(x1, -127.f));
  const uint64_t t = add2(xv, f2pack(kShift, kShift));
  const uint64_t n = add2(t, f2pack(-kShift, -kShift));  // round(x), exact
  const uint64_t f = fma2(n, f2pack(-1.f, -1.f), xv);    // x - round(x)
  uint64_t q = fma2(f2pack(0.055171605f, 0.055171605f), f, f2pack(0.24261111f, 0.24261111f));
  q = fma2(q, f, f2pack(0.69326097f, 0.69326097f));
  q = fma2(q, f, f2pack(0.99992806f, 0.99992806f));
  float t0, t1;
  f2unpack(t, t0, t1);
  // The low bits of t hold round(x) + 0x4B400000; shifted into the exponent
  // field the 0x4B400000 part vanishes and +127 << 23 biases it.
  const float s0 = __uint_as_float((__float_as_uint(t0) << 23) + 0x3F800000u);
  const float s1 = __uint_as_float((__float_as_uint(t1) << 23) + 0x3F800000u);
  return mul2(q, f2pack(s0, s1));
}

struct Params {
  const int4* qtiles;  // per piece: {qt, seg_begin, seg_count, n_ktiles}
  const int2* segs;    // {kt_begin, (count << 1) | partial}
  const int2* piece_meta;  // per piece: {bh, partial slot or -1}
  int n_entries, n_segs, n_items, n_qt, n_kt, n_bh;
  int Lq, Lk;
  float scale, c2;
  __nv_bfloat16* o;    // [B*H, Lq, d]
  float* lse;          // [B*H, Lq]
  float* part;         // [slots, 128, d] unnormalised partial O
  float2* ml;          // [slots, 128] {running max (log2), sum}
  unsigned* err;
  unsigned* item_ctr;
  unsigned long long wait_limit_ns;
  int stall_test;  // the MMA warp first waits on a phase that nothing completes
};
using Cursor = pipe::Cursor<Params>;

__global__ void __launch_bounds__(kThreads, 1)
attn_cache_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
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
    for (uint32_t s = 0; s < NK; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_KEMPTY + s), 1);
    }
    for (uint32_t s = 0; s < 2; ++s) {
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_VEMPTY + s), 1);
      mbar_init(bar(B_SFULL + s), 1);
      mbar_init(bar(B_PFULL + s), 2 * BM);
      mbar_init(bar(B_PVD + s), 1);
    }
    mbar_init(bar(B_AFREE), 2 * BM);
    mbar_init(bar(B_DRAIN), 1);
    mbar_init(bar(B_DRAIN2), 1);
    for (int i = 0; i < 4; ++i) mbar_init(bar(B_XSUM + i), 64);
    for (uint32_t i = 0; i < kRing; ++i) {
      mbar_init(bar(B_IFULL + i), 1);
      mbar_init(bar(B_IEMPTY + i), kRingReaders);
    }
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tm_q);
    tma_prefetch_map(&tm_k);
    tma_prefetch_map(&tm_v);
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
      uint32_t q_armed = 0, k_issued = 0, v_issued = 0;
      bool ok = true;
      while (c.valid && ok) {
        if (c.j == 0) {
          if (c.item_idx > 0) ok = wait_bar(bar(B_QEMPTY), (c.item_idx - 1) & 1, p, abort_flag);
          if (!ok) break;
          mbar_expect_tx(bar(B_QFULL), kStage);
          ++q_armed;
          const int y = c.qt * BM;
          tma_load_3d(base + SM_Q, &tm_q, bar(B_QFULL), 0, y, c.bh);
          tma_load_3d(base + SM_Q + kHalf, &tm_q, bar(B_QFULL), 64, y, c.bh);
        }
        const int y = c.kt * BN;
        const uint32_t sk = c.t % NK, uk = c.t / NK;
        if (c.t >= NK) ok = wait_bar(bar(B_KEMPTY + sk), (uk - 1) & 1u, p, abort_flag);
        if (!ok) break;
        mbar_expect_tx(bar(B_KFULL + sk), kStage);
        ++k_issued;
        tma_load_3d(base + SM_K + sk * kStage, &tm_k, bar(B_KFULL + sk), 0, y, c.bh);
        tma_load_3d(base + SM_K + sk * kStage + kHalf, &tm_k, bar(B_KFULL + sk), 64, y, c.bh);
        const uint32_t sv = c.t & 1u, uv = c.t >> 1;
        if (c.t >= NV) ok = wait_bar(bar(B_VEMPTY + sv), (uv - 1) & 1u, p, abort_flag);
        if (!ok) break;
        mbar_expect_tx(bar(B_VFULL + sv), kStage);
        ++v_issued;
        tma_load_3d(base + SM_V + sv * kStage, &tm_v, bar(B_VFULL + sv), 0, y, c.bh);
        tma_load_3d(base + SM_V + sv * kStage + kHalf, &tm_v, bar(B_VFULL + sv), 64, y, c.bh);
        c.next(p, ring, kProducer);
      }
      if (!ok || *abort_flag) {
        if (q_armed) drain_wait(bar(B_QFULL), (q_armed - 1) & 1u);
        for (uint32_t s = 0; s < NK; ++s) {
          const uint32_t n = (k_issued + NK - 1 - s) / NK;
          if (n) drain_wait(bar(B_KFULL + s), (n - 1) & 1u);
        }
        for (uint32_t s = 0; s < NV; ++s) {
          const uint32_t n = (v_issued + NV - 1 - s) / NV;
          if (n) drain_wait(bar(B_VFULL + s), (n - 1) & 1u);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA ----
    // Each MMA warp runs its loop in uniform control flow; one elected lane
    // issues each MMA and commit.
    {
      bool ok = true;
      auto wait_w = [&](uint32_t b_, uint32_t par_) -> bool {
        return __all_sync(0xffffffffu, wait_bar(b_, par_, p, abort_flag));
      };
      const uint64_t q_desc = sdesc_sw128(base + SM_Q, 16, 1024);
      const uint64_t k_desc = sdesc_sw128(base + SM_K, 16, 1024);     // K-major, stage 0
      const uint64_t v_desc = sdesc_sw128(base + SM_V, kHalf, 1024);  // MN-major, stage 0
      auto issue_s = [&](const Cursor& c) -> bool {
        const uint32_t b = c.t & 1u, sk = c.t % NK;
        if (c.j == 0 && !wait_w(bar(B_QFULL), c.item_idx & 1)) return false;
        // Buffer b last held tile t-2, whose P PV(t-2) reads: S(t) waits
        // until those MMAs (warp 2's) have completed; MMAs of different warps
        // are ordered only through completions.
        if (c.t >= 2 && !wait_w(bar(B_PVD + b), ((c.t >> 1) - 1) & 1u)) return false;
        if (!wait_w(bar(B_KFULL + sk), (c.t / NK) & 1u)) return false;
        tc_fence_after();
        const uint64_t kb = k_desc + sk * (kStage >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
          mma_ss_elect(tmem + b * 128u, q_desc + off, kb + off, IDESC_S, kk > 0);
        }
        mma_commit_elect(bar(B_SFULL + b));
        mma_commit_elect(bar(B_KEMPTY + sk));
        if (c.j == c.n - 1) mma_commit_elect(bar(B_QEMPTY));
        return true;
      };
      auto issue_pv = [&](const Cursor& c) -> bool {
        const uint32_t b = c.t & 1u;
        if (c.j == 0 && c.item_idx > 0 &&
            !wait_w(bar(B_AFREE), (c.item_idx - 1) & 1))
          return false;
        if (!wait_w(bar(B_PFULL + b), (c.t >> 1) & 1u)) return false;
        if (!wait_w(bar(B_VFULL + b), (c.t >> 1) & 1u)) return false;
        tc_fence_after();
        const uint64_t vb = v_desc + b * (kStage >> 4);
        const uint32_t first = c.j == 0 ? 0u : 1u;
        // O_a += P[:, 0:64] V[0:64], O_b += P[:, 64:128] V[64:128]: 4 steps of
        // 16 keys each. The bf16 P of keys [64 h, 64 h + 64) is packed into
        // buffer columns [64 h, 64 h + 32), the start of the S columns that
        // softmax warpgroup h itself read.
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks)
          mma_ts_elect(tmem + TM_O + (ks >> 2) * 128u,
                 tmem + b * 128u + (ks >> 2) * 64u + (ks & 3) * 8u,
                 vb + ((ks * 2048) >> 4), IDESC_PV, first | ((ks & 3) > 0));
        mma_commit_elect(bar(B_VEMPTY + b));
        mma_commit_elect(bar(B_PVD + b));
        return true;
      };
      // Warp 1 issues S(t), warp 2 PV(t); S(t+2) waits for PV(t) to complete.
      const bool s_warp = warp == 1;
      Cursor c;
      c.start(p, ring, kConsumerWarp);
      // Failure-detection test: wait on the drain barrier's first phase,
      // which nothing completes before this warp's own drain commit, so the
      // bounded wait runs out and the abort path below is taken.
      if (p.stall_test && s_warp)
        ok = __all_sync(0xffffffffu, wait_bar(bar(B_DRAIN), 0u, p, abort_flag));
      while (c.valid && ok) {
        ok = s_warp ? issue_s(c) : issue_pv(c);
        c.next(p, ring, kConsumerWarp);
      }
      if (__any_sync(0xffffffffu, !ok || *abort_flag)) {
        const uint32_t db = bar(s_warp ? B_DRAIN : B_DRAIN2);
        mma_commit_elect(db);
        drain_wait(db, 0);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ----------------------------------------------------------- softmax ----
    // Warps 4-7 take keys [0, 64) of every 128-key tile, warps 8-11 keys
    // [64, 128) (one row per thread, TMEM lane quarter q for warps 4+q and
    // 8+q). Each warpgroup keeps its own running max and sum for its half
    // and accumulates into its own O (O_a or O_b), so the two never wait for
    // each other inside an item; the epilogue merges the halves.
    const int hw = (warp - 4) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t tl = tmem + (uint32_t(q4 * 32) << 16);
    const uint32_t my_o = TM_O + 128u * hw;
    float* const xsum = reinterpret_cast<float*>(base_ptr + SM_XCHG);  // [2 (m, l)][2][128]
    Cursor c;
    c.start(p, ring, kConsumerWarp);
    float m_ref = -CUDART_INF_F, l = 0.f;
    int grow = 0;
    bool ok = true;
    while (c.valid) {
      if (c.j == 0) {
        grow = c.qt * BM + r;
        m_ref = -CUDART_INF_F;
        l = 0.f;
      }
      const uint32_t b = c.t & 1u;
      ok = wait_bar(bar(B_SFULL + b), (c.t >> 1) & 1u, p, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t sa[32], sb[32];
      tmem_ld32(tl + b * 128u + 64u * hw, sa);
      tmem_ld32(tl + b * 128u + 64u * hw + 32u, sb);
      tmem_wait_ld();
      float s[64];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        s[i] = __uint_as_float(sa[i]);
        s[32 + i] = __uint_as_float(sb[i]);
      }
      if (c.partial) {  // the tile holding key Lk - 1: keys past Lk are not in the prefix
        const int k0 = c.kt * BN + 64 * hw;
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (k0 + i >= p.Lk) s[i] = -CUDART_INF_F;
      }
      float m8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) m8[i] = s[i];
#pragma unroll
      for (int i = 8; i < 64; ++i) m8[i & 7] = fmaxf(m8[i & 7], s[i]);
#pragma unroll
      for (int w2 = 4; w2 > 0; w2 >>= 1)
#pragma unroll
        for (int i = 0; i < w2; ++i) m8[i] = fmaxf(m8[i], m8[i + w2]);
      const float mxs = m8[0] * p.c2;  // -inf while every key of this half is masked
      float alpha = 1.f;
      bool need = false;
      if (m_ref == -CUDART_INF_F) {
        m_ref = mxs;  // first keys of this half: nothing accumulated yet (l = 0)
      } else if (mxs > m_ref + kTau) {
        alpha = ex2(m_ref - mxs);
        m_ref = mxs;
        need = true;
      }
      // Each warp decides for its own rows and scales only its own O.
      if (__any_sync(0xffffffffu, need)) {
        l *= alpha;
        // This O holds PV(t-1); wait for it. (PV(t-3), the previous phase of
        // that barrier, completed before S(t-1) was issued.)
        ok = wait_bar(bar(B_PVD + ((c.t - 1) & 1u)), ((c.t - 1) >> 1) & 1u, p, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          uint32_t a[32];
          tmem_ld32(tl + my_o + 32u * q, a);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) a[i] = __float_as_uint(__uint_as_float(a[i]) * alpha);
          tmem_st32(tl + my_o + 32u * q, a);
        }
        tmem_wait_st();
      }
      // e = 2^(c2 s - m) in packed pairs (m = 0 while the half is all
      // masked, so that e = 0 there); bf16 P over the first 32 of the S
      // columns this warp has just read (never the other warpgroup's).
      const float mref_use = m_ref == -CUDART_INF_F ? 0.f : m_ref;
      const uint64_t c2v = f2pack(p.c2, p.c2), mv = f2pack(-mref_use, -mref_use);
      uint64_t la = 0, lb = 0;
      uint32_t pp[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        float x0, x1;
        f2unpack(fma2(f2pack(s[2 * i], s[2 * i + 1]), c2v, mv), x0, x1);
        // A quarter of the pairs on the FMA pipe, the rest on MUFU.
        float e0, e1;
        if ((i & 3) == 3) {
          f2unpack(ex2_fma2(x0, x1), e0, e1);
        } else {
          e0 = ex2(x0);
          e1 = ex2(x1);
        }
        if (i & 1) lb = add2(lb, f2pack(e0, e1));
        else la = add2(la, f2pack(e0, e1));
        pp[i] = pack_bf16(e0, e1);
      }
      {
        float u0, u1;
        f2unpack(add2(la, lb), u0, u1);
        l += u0 + u1;
      }
      tmem_st32(tl + b * 128u + 64u * hw, pp);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_PFULL + b));

      if (c.j == c.n - 1) {
        // ------------------------------------------------------ epilogue --
        // PV(t) done; PV(t-2), the previous phase of this barrier, completed
        // before S(t) was issued.
        ok = wait_bar(bar(B_PVD + (c.t & 1u)), (c.t >> 1) & 1u, p, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) break;
        xsum[hw * BM + r] = m_ref;
        xsum[(2 + hw) * BM + r] = l;
        mbar_arrive(bar(B_XSUM + q4));
        ok = wait_bar(bar(B_XSUM + q4), c.item_idx & 1, p, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) break;
        // Merge the halves: M = max(m_a, m_b), w = 2^(m - M) (0 for an
        // all-masked half), L = w_a l_a + w_b l_b.
        const float m_a = hw == 0 ? m_ref : xsum[r], m_b = hw == 1 ? m_ref : xsum[BM + r];
        const float l_a = hw == 0 ? l : xsum[2 * BM + r], l_b = hw == 1 ? l : xsum[3 * BM + r];
        const float M = fmaxf(m_a, m_b);
        const float w_a = m_a == -CUDART_INF_F ? 0.f : ex2(m_a - M);
        const float w_b = m_b == -CUDART_INF_F ? 0.f : ex2(m_b - M);
        const float lt = w_a * l_a + w_b * l_b;
        tc_fence_after();
        const bool row_ok = grow < p.Lq;
        const int slot = p.piece_meta[c.item].y;  // -1: this piece is the whole item
        const bool split = slot >= 0;
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        const float sa_ = split ? w_a : w_a * inv, sb_ = split ? w_b : w_b * inv;
        // This warpgroup writes head-dim columns [64 hw, 64 hw + 64).
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
          const uint32_t col = 64u * hw + 32u * cc;
          uint32_t oa[32], ob[32];
          tmem_ld32(tl + TM_O + col, oa);
          tmem_ld32(tl + TM_O + 128u + col, ob);
          tmem_wait_ld();
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            v[i] = fmaf(__uint_as_float(oa[i]), sa_, __uint_as_float(ob[i]) * sb_);
          if (!split) {
            if (row_ok) {
              uint4* go = reinterpret_cast<uint4*>(p.o + (size_t(c.bh) * p.Lq + grow) * D + col);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                go[i] = make_uint4(pack_bf16(v[8 * i], v[8 * i + 1]),
                                   pack_bf16(v[8 * i + 2], v[8 * i + 3]),
                                   pack_bf16(v[8 * i + 4], v[8 * i + 5]),
                                   pack_bf16(v[8 * i + 6], v[8 * i + 7]));
            }
          } else {
            // Unnormalised partial of this piece relative to M, for every
            // row of the tile (rows past Lq are never combined).
            float4* dst = reinterpret_cast<float4*>(p.part + (size_t(slot) * BM + r) * D + col);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          }
        }
        tc_fence_before();
        mbar_arrive(bar(B_AFREE));
        if (hw == 0) {
          if (split)
            p.ml[size_t(slot) * BM + r] = make_float2(M, lt);
          else if (row_ok)
            p.lse[size_t(c.bh) * p.Lq + grow] =
                lt > 0.f ? (M + log2f(lt)) * 0.69314718055994531f : -CUDART_INF_F;
        }
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

// Combines the pieces of each split item, row by row: with per-piece
// running max m_s (log2 units of the scaled score), sum l_s and unnormalised
// partial O_s,
//   M = max m_s,  w_s = 2^(m_s - M),  O = sum w_s O_s / sum w_s l_s,
//   LSE = (M + log2 sum w_s l_s) ln 2.
// One warp per (split item, row of its query tile), 4 head-dim columns per
// lane. splits[i] = {bh, qt, first slot, slot count}.
__global__ void __launch_bounds__(256)
attn_cache_combine_kernel(const float* __restrict__ part, const float2* __restrict__ ml,
                          const int4* __restrict__ splits, int n_splits, int n_slots,
                          __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int n_bh,
                          int Lq, unsigned* err) {
  const int lane = threadIdx.x & 31;
  const long long n_rows = (long long)n_splits * BM;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < n_rows;
       w += warps) {
    const int4 sp = splits[w / BM];
    const int r = int(w % BM);
    const int bh = sp.x, i = sp.y * BM + r;
    if (bh < 0 || bh >= n_bh || sp.z < 0 || sp.w < 1 || sp.z + sp.w > n_slots) {
      if (lane == 0) atomicOr(err, kErrBounds);
      continue;
    }
    if (i >= Lq) continue;
    float M = -CUDART_INF_F;
    for (int s = sp.z; s < sp.z + sp.w; ++s) M = fmaxf(M, ml[size_t(s) * BM + r].x);
    float lsum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = sp.z; s < sp.z + sp.w; ++s) {
      const float2 v = ml[size_t(s) * BM + r];
      const float ws = v.x == -CUDART_INF_F ? 0.f : exp2f(v.x - M);
      lsum += ws * v.y;
      const float4 pv = reinterpret_cast<const float4*>(part + (size_t(s) * BM + r) * D)[lane];
      acc.x += ws * pv.x;
      acc.y += ws * pv.y;
      acc.z += ws * pv.z;
      acc.w += ws * pv.w;
    }
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
    uint2 packed;
    packed.x = pack_bf16(acc.x * inv, acc.y * inv);
    packed.y = pack_bf16(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2*>(o + (size_t(bh) * Lq + i) * D)[lane] = packed;
    if (lane == 0)
      lse[size_t(bh) * Lq + i] =
          lsum > 0.f ? (M + log2f(lsum)) * 0.69314718055994531f : -CUDART_INF_F;
  }
}

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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

// [BH, rows_alloc, 128] bf16 with `rows` readable rows per (b, h): the map's
// row extent is `rows`, so reads past it are zero-filled.
static bool make_map(CUtensorMap* m, const void* ptr, int rows, int rows_alloc, int BH) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(rows), cuuint64_t(BH)};
  cuuint64_t strides[2] = {cuuint64_t(D) * 2, cuuint64_t(rows_alloc) * D * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace cache

int launch_cache_sm100(const CacheArgs& a, const CacheWork& cw, int num_sms) {
  using namespace cache;
  const int BH = a.B * a.H;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.q, a.Lq, a.Lq, BH) || !make_map(&mk, a.k, a.Lk, a.Lcache, BH) ||
      !make_map(&mv, a.v, a.Lk, a.Lcache, BH))
    return JVP_ERR_LAUNCH_FAILED;
  Params p;
  p.qtiles = cw.w.qtiles;
  p.segs = cw.w.segs;
  p.piece_meta = cw.meta;
  p.n_entries = cw.w.n_qtiles;
  p.n_segs = cw.w.n_segs;
  p.n_items = cw.w.n_qtiles;
  p.n_qt = (a.Lq + BM - 1) / BM;
  p.n_kt = (a.Lk + BN - 1) / BN;
  p.n_bh = BH;
  p.Lq = a.Lq;
  p.Lk = a.Lk;
  p.scale = a.scale;
  p.c2 = a.scale * 1.4426950408889634f;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.lse = a.lse;
  p.part = a.part;
  p.ml = reinterpret_cast<float2*>(a.ml);
  p.err = a.err;
  p.item_ctr = a.item_ctr;
  p.wait_limit_ns = a.wait_limit_ns;
  p.stall_test = a.stall_test ? 1 : 0;
  if (p.n_items < 1 || (cw.n_slots > 0 && (!p.part || !p.ml))) return JVP_ERR_LAUNCH_FAILED;
  static std::mutex attr_mu;
  static bool attr_done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return JVP_ERR_LAUNCH_FAILED;
  {
    std::lock_guard<std::mutex> lk(attr_mu);
    if (!attr_done[dev]) {
      if (cudaFuncSetAttribute(attn_cache_sm100_kernel,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kSmemBytes) != cudaSuccess)
        return JVP_ERR_LAUNCH_FAILED;
      attr_done[dev] = true;
    }
  }
  const int grid = p.n_items < num_sms ? p.n_items : num_sms;
  if (!a.item_ctr || cudaMemsetAsync(a.item_ctr, 0, sizeof(unsigned), a.stream) != cudaSuccess)
    return JVP_ERR_LAUNCH_FAILED;
  attn_cache_sm100_kernel<<<grid, kThreads, kSmemBytes, a.stream>>>(mq, mk, mv, p);
  if (cudaGetLastError() != cudaSuccess) return JVP_ERR_LAUNCH_FAILED;
  if (cw.n_splits > 0) {
    const long long rows = (long long)cw.n_splits * BM;
    const long long blocks = (rows + 7) / 8;  // 8 warps per block
    const int cgrid = int(blocks < 8LL * num_sms ? blocks : 8LL * num_sms);
    attn_cache_combine_kernel<<<cgrid, 256, 0, a.stream>>>(p.part, p.ml, cw.splits, cw.n_splits,
                                                           cw.n_slots, p.o, p.lse, BH, a.Lq,
                                                           a.err);
    if (cudaGetLastError() != cudaSuccess) return JVP_ERR_LAUNCH_FAILED;
  }
  return JVP_OK;
}

}  // namespace jvp
