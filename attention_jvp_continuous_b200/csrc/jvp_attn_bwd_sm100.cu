// Backward pass of masked softmax attention for B200 (sm_100a): the gradient
// of sum <G, O> with O = softmax(c QK^T + M) V (Causal-rCM report, Eq. 42;
// the consistency loss is differentiated through the primal output only,
// Appendix A). With P = exp(c QK^T - LSE) (the forward's LSE), D_i = <g_i, o_i>:
//   dP = G V^T,  dS = P o (dP - D),  gQ = c dS K,  gK = c dS^T Q,  gV = P^T G.
//
// Two persistent tcgen05 kernels over the same admissible-tile work lists:
//  * dQ pass (query-stationary, 128 query rows per item, 128-key tiles):
//      S = Q K^T, dP = G V^T   (N = 128, both operands in shared memory; two
//                               S parts and one dP part in TMEM)
//      softmax warps: P, dS    (one row per thread, bf16 dS back to TMEM)
//      gQ += dS K              (A = dS in TMEM, N = 128, accumulator in TMEM)
//    and it writes -LSE2 and -D_i per row pair to a scratch vector for the
//    second pass.
//  * dK/dV pass (key-stationary, 128 keys per item, 64-query tiles):
//      S^T = K Q^T, dP^T = V G^T (both operands in shared memory: TMEM holds
//                               the two accumulators and two S/dP buffers)
//      softmax warps: P^T, dS^T (one key per thread; per-query LSE and D
//                               from the scratch, copied into shared memory
//                               with each Q tile)
//      gV += P^T G, gK += dS^T Q (A in TMEM, N = 128)
// Warp roles: warp 0 TMA, warps 1 and 2 issue MMAs (whole warps, one
// elected lane issuing), warps 4-11 two warpgroups taking half of each
// tile's columns (64 of 128 keys in the dQ pass, 32 of 64 queries in the
// dK/dV pass). Each warpgroup writes its bf16 operands into the TMEM columns
// it has just read itself, so no exchange between the warpgroups is needed.
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
namespace bwd {

using namespace jvp::ptx;
using pipe::drain_wait;
using pipe::ItemRing;
using pipe::kConsumerWarp;
using pipe::kProducer;
using pipe::kRing;
using pipe::wait_bar;

constexpr int BR = 128;  // stationary rows per item (TMEM lanes)
constexpr int D = 128;
constexpr int kThreads = 384;
// Streamed rows per tile: 128 keys (dQ pass), 64 queries (dK/dV pass).
template <bool kKV> constexpr int kBT = kKV ? 64 : 128;

constexpr uint32_t kRHalf = BR * 128;  // 16 KB: 128 rows x 64 head-dim columns
template <bool kKV> constexpr uint32_t kTHalf = kBT<kKV> * 128;  // rows x 64 columns
template <bool kKV> constexpr uint32_t kTile = 2 * kTHalf<kKV>;   // one streamed operand
// Readers of the work-item ring: issuer A's two cursors, issuer B's one (dQ)
// or two (dK/dV), 8 softmax warps.
template <bool kKV> constexpr uint32_t kReaders = (kKV ? 4 : 3) + 8;

// Four MMAs into one accumulator behind a single elect.sync: the whole warp
// runs the block, the elected lane issues all four (in order). acc0 is the
// first one's enable-input-d; the other three accumulate.
__device__ __forceinline__ void mma_ts4_elect(uint32_t d_tmem, uint32_t a0, uint32_t a1,
                                              uint32_t a2, uint32_t a3, uint64_t b0, uint64_t b1,
                                              uint64_t b2, uint64_t b3, uint32_t idesc,
                                              uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred e, p, q;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %10, 0;\n\t"
      "setp.ne.b32 q, %11, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %5, %9, p;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], %6, %9, q;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%3], %7, %9, q;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%4], %8, %9, q;\n\t}" ::"r"(d_tmem),
      "r"(a0), "r"(a1), "r"(a2), "r"(a3), "l"(b0), "l"(b1), "l"(b2), "l"(b3), "r"(idesc),
      "r"(acc0), "r"(1u)
      : "memory");
}
__device__ __forceinline__ void mma_ss4_elect(uint32_t d_tmem, uint64_t a0, uint64_t a1,
                                              uint64_t a2, uint64_t a3, uint64_t b0, uint64_t b1,
                                              uint64_t b2, uint64_t b3, uint32_t idesc,
                                              uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred e, p, q;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %10, 0;\n\t"
      "setp.ne.b32 q, %11, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %5, %9, p;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %6, %9, q;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %7, %9, q;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %8, %9, q;\n\t}" ::"r"(d_tmem),
      "l"(a0), "l"(a1), "l"(a2), "l"(a3), "l"(b0), "l"(b1), "l"(b2), "l"(b3), "r"(idesc),
      "r"(acc0), "r"(1u)
      : "memory");
}

// Plain bulk copy global -> shared, completing on an mbarrier (no tensor map,
// no multicast): dst and src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Shared memory: the item's two stationary operands (A0, A1: Q and G, or K
// and V, 32 KB each), then the streamed operands in two rings X and Y, and
// in the dK/dV pass each X stage's per-query slice of the scratch (W: 32 row
// pairs {-LSE2, -LSE2, -D, -D}, 512 B), loaded with the stage. Stages: dQ
// pass (32 KB tiles of 128 keys), K feeds S(t) and gQ(t), S one tile ahead
// of gQ: 3; V feeds dP only: 2. dK/dV pass (16 KB tiles of 64 queries): Q
// and G feed one first and one accumulating batch each, the first batch one
// tile ahead of the accumulating one: 4 each.
template <bool kKV>
struct Layout {
  static constexpr uint32_t NX = kKV ? 4 : 3;  // dQ: K    dK/dV: Q
  static constexpr uint32_t NY = kKV ? 4 : 2;  // dQ: V    dK/dV: G
  static constexpr uint32_t A0 = 0;
  static constexpr uint32_t A1 = 2 * kRHalf;
  static constexpr uint32_t X = 4 * kRHalf;
  static constexpr uint32_t Y = X + NX * kTile<kKV>;
  static constexpr uint32_t W = Y + NY * kTile<kKV>;
  static constexpr uint32_t BAR = W + (kKV ? NX * 512 : 0);  // 224 KB (dQ) / 194 KB (dK/dV)
  static constexpr uint32_t TMEM_SLOT = BAR + 8 * 44;
  static constexpr uint32_t ABORT = TMEM_SLOT + 4;
  static constexpr uint32_t RING = ABORT + 4;
  static constexpr uint32_t kBytes = BAR + 512 + 1024;  // + alignment slack
};
static_assert(Layout<true>::kBytes <= 232448 && Layout<false>::kBytes <= 232448,
              "shared memory over the per-block limit");

enum : uint32_t {
  B_AF = 0,      // stationary operands ready (TMA bytes)
  B_AE = 1,      // stationary operands may be overwritten (2 issuers)
  B_XF = 2,      // 6
  B_XE = 8,      // 6 (dK/dV pass: releases the X and the Y stage)
  B_YF = 14,     // 5
  B_YE = 19,     // 4 (dQ pass only)
  B_SF = 23,     // 3: S and dP of a buffer complete (one commit per issuer)
  B_PF = 26,     // 3: bf16 operands written by the softmax warps
  B_DR = 29,     // dQ pass: the softmax warps have read the dP part
  B_MD = 30,     // accumulating MMAs of an item's last tile complete
  B_CF = 31,     // accumulators read by the epilogue
  B_DRAIN = 32,  // 2: one per issuer
  B_IF = 34,     // 4: work-item ring
  B_IE = 38,     // 4
  kNumBars = 42
};
static_assert(Layout<false>::NY <= B_SF - B_YE, "Y-empty slots");
static_assert(Layout<false>::NX <= B_XE - B_XF && Layout<false>::NX <= B_YF - B_XE, "X slots");
static_assert(Layout<true>::NX == Layout<true>::NY, "dK/dV pass: X and Y stages pair up");
static_assert(kNumBars <= 44, "barrier slots");
static_assert(Layout<false>::RING + 16 <= Layout<false>::BAR + 512, "barrier area overflow");

// TMEM columns. dQ pass: two 128-column S parts (part b at 128 b) and one
// dP part at 256, since the softmax warps are done with dP as soon as they
// have loaded it, while an S part holds dS until the accumulating MMAs have
// read it; gQ at 384. dK/dV pass: two buffers (buffer b at 128 b: S^T at +0,
// dP^T at +64), gV at 256 and gK at 384.
template <bool kKV> constexpr uint32_t kBufs = 2;
template <bool kKV> __device__ __forceinline__ uint32_t s_col(uint32_t b) { return 128u * b; }
template <bool kKV> __device__ __forceinline__ uint32_t dp_col(uint32_t b) {
  return kKV ? 128u * b + 64u : 256u;
}
template <bool kKV> constexpr uint32_t kC0 = kKV ? 256u : 384u;  // gV, or gQ
constexpr uint32_t TM_C1 = 384;  // gK

// First MMAs: 128 x 128 (dQ pass) or 128 x 64 (dK/dV pass), K-major B.
template <bool kKV>
constexpr uint32_t kIdescFirst = ptx::idesc_bf16(BR, kBT<kKV>, false, false);
constexpr uint32_t IDESC_MN = ptx::idesc_bf16(BR, D, false, true);  // 128 x 128, MN-major B

struct Params {
  const int4* qtiles;  // work entries {outer tile, seg_begin, seg_count, inner tiles}
  const int2* segs;
  int n_entries, n_segs, n_items, n_qt, n_kt;  // n_qt: outer tiles, n_kt: inner tiles
  int L;
  jvp_mask_desc mask;
  int Lp;  // L rounded up to whole 128-row tiles: row stride of the scratch
  float scale, c2;
  const float* lse;     // forward LSE (natural log)
  // Scratch [B*H, Lp / 2] of one float4 per row pair (2m, 2m+1):
  // {-LSE2_2m, -LSE2_2m+1, -D_2m, -D_2m+1}, LSE2 = LSE log2(e), D_i = <g_i, o_i>;
  // written by the dQ pass (rows past L: LSE2 = +inf, D = 0), read by the
  // dK/dV pass as packed fp32 pairs.
  float* sd;
  const __nv_bfloat16* q;  // query rows
  const __nv_bfloat16* g;  // cotangent rows, for D (dQ pass)
  const __nv_bfloat16* o;  // forward output, for D (dQ pass)
  __nv_bfloat16* out0;     // gQ (dQ pass) or gK (dK/dV pass)
  __nv_bfloat16* out1;     // gV (dK/dV pass)
  unsigned* err;
  unsigned* item_ctr;
  unsigned long long wait_limit_ns;
  int stall_test;  // the MMA warp first waits on a phase that nothing completes
};
using Cursor = pipe::Cursor<Params>;

// Ring stage of a cursor's tile t and the parity of its use, kept in step
// with the cursor (t % N and (t / N) & 1 without the division).
struct Stage {
  uint32_t s = 0, ph = 0;
  __device__ void step(uint32_t n) {
    if (++s == n) {
      s = 0;
      ph ^= 1u;
    }
  }
};

// MMA issue is split over two warps (one elected lane of each issues), since
// one lane issues at most about one tcgen05.mma per ~47 cycles while a
// 128 x 64 x 16 MMA takes 32. MMAs of different warps are ordered only
// through completions, so the warp that reads a TMEM part in tile t's
// accumulating MMAs is the one that overwrites it at tile t+2:
//   dQ pass:    issuer A (warp 1): gQ(t) once the softmax warps have written
//               tile t's dS into S part t&1, then S(t+2) = A0 X(t+2)^T into
//               that part; issuer B (warp 2): dP(t) = A1 Y(t)^T into the one
//               dP part once the softmax warps have loaded dP(t-1) from it.
//   dK/dV pass: issuer A: gV(t) (P^T, S part) then S^T(t+2); issuer B:
//               gK(t) (dS^T, dP part) then dP^T(t+2).
// One thread's MMAs run in issue order; every hand-over between the issuers
// and the other roles goes through an mbarrier.
template <bool kKV>
__global__ void __launch_bounds__(kThreads, 1)
bwd_kernel(const __grid_constant__ CUtensorMap tm_a0, const __grid_constant__ CUtensorMap tm_a1,
           const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_y,
           const __grid_constant__ Params p) {
  // dQ pass:  A0 = Q, A1 = G (stationary);  X = K, Y = V (rings).
  // dK/dV:    A0 = K, A1 = V (stationary);  X = Q, Y = G.
  using LY = Layout<kKV>;
  constexpr uint32_t NX = LY::NX, NY = LY::NY;
  constexpr int BT = kBT<kKV>;
  constexpr uint32_t kTH = kTHalf<kKV>, kTL = kTile<kKV>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  auto bar = [&](uint32_t slot) { return base + LY::BAR + 8u * slot; };
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(base_ptr + LY::ABORT);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    // dQ: the 256 softmax threads store Q / G rows and arrive; dK/dV: TMA bytes.
    mbar_init(bar(B_AF), 1);
    mbar_init(bar(B_AE), 2);
    // dK/dV pass: a stage pair (Q and G of one tile) is released and an
    // item's accumulation is complete once both issuers have committed
    // (each runs half of the accumulation).
    for (uint32_t s = 0; s < NX; ++s) {
      mbar_init(bar(B_XF + s), 1);
      mbar_init(bar(B_XE + s), kKV ? 2 : 1);
    }
    for (uint32_t s = 0; s < NY; ++s) {
      mbar_init(bar(B_YF + s), 1);
      if (!kKV) mbar_init(bar(B_YE + s), 1);
    }
    for (uint32_t b = 0; b < kBufs<kKV>; ++b) {
      mbar_init(bar(B_SF + b), 2);
      mbar_init(bar(B_PF + b), 2 * BR);
    }
    mbar_init(bar(B_DR), 2 * BR);
    for (int b = 0; b < 2; ++b) mbar_init(bar(B_DRAIN + b), 1);
    mbar_init(bar(B_MD), kKV ? 2 : 1);
    mbar_init(bar(B_CF), 2 * BR);
    for (uint32_t i = 0; i < kRing; ++i) {
      mbar_init(bar(B_IF + i), 1);
      mbar_init(bar(B_IE + i), kReaders<kKV>);
    }
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tm_a0);
    tma_prefetch_map(&tm_a1);
    tma_prefetch_map(&tm_x);
    tma_prefetch_map(&tm_y);
  }
  if (warp == 1) {
    tmem_alloc(base + LY::TMEM_SLOT, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(base_ptr + LY::TMEM_SLOT);
  const ItemRing ring{bar(B_IF), bar(B_IE),
                      reinterpret_cast<volatile int*>(base_ptr + LY::RING), abort_flag};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA ----
    if (lane == 0) {
      Cursor c;
      c.start(p, ring, kProducer);
      uint32_t a_armed = 0, x_issued = 0, y_issued = 0;
      bool ok = true;
      while (c.valid && ok) {
        if (c.j == 0) {
          if (c.item_idx > 0) ok = wait_bar(bar(B_AE), (c.item_idx - 1) & 1, p, abort_flag);
          if (!ok) break;
          mbar_expect_tx(bar(B_AF), 4 * kRHalf);
          ++a_armed;
          const int y = c.qt * BR;
          tma_load_3d(base + LY::A0, &tm_a0, bar(B_AF), 0, y, c.bh);
          tma_load_3d(base + LY::A0 + kRHalf, &tm_a0, bar(B_AF), 64, y, c.bh);
          tma_load_3d(base + LY::A1, &tm_a1, bar(B_AF), 0, y, c.bh);
          tma_load_3d(base + LY::A1 + kRHalf, &tm_a1, bar(B_AF), 64, y, c.bh);
        }
        const int y = c.kt * BT;
        const uint32_t sx = c.t % NX, ux = c.t / NX;
        if (c.t >= NX) ok = wait_bar(bar(B_XE + sx), (ux - 1) & 1u, p, abort_flag);
        if (!ok) break;
        mbar_expect_tx(bar(B_XF + sx), kKV ? kTL + 512u : kTL);
        ++x_issued;
        if (kKV)
          bulk_load(base + LY::W + sx * 512u, p.sd + (size_t(c.bh) * p.Lp + y) * 2, 512u,
                    bar(B_XF + sx));  // this tile's 64 queries: 16-byte aligned (y % 64 == 0)
        tma_load_3d(base + LY::X + sx * kTL, &tm_x, bar(B_XF + sx), 0, y, c.bh);
        tma_load_3d(base + LY::X + sx * kTL + kTH, &tm_x, bar(B_XF + sx), 64, y, c.bh);
        const uint32_t sy = c.t % NY, uy = c.t / NY;
        if (!kKV && c.t >= NY) ok = wait_bar(bar(B_YE + sy), (uy - 1) & 1u, p, abort_flag);
        if (!ok) break;
        mbar_expect_tx(bar(B_YF + sy), kTL);
        ++y_issued;
        tma_load_3d(base + LY::Y + sy * kTL, &tm_y, bar(B_YF + sy), 0, y, c.bh);
        tma_load_3d(base + LY::Y + sy * kTL + kTH, &tm_y, bar(B_YF + sy), 64, y, c.bh);
        c.next(p, ring, kProducer);
      }
      if (!ok || *abort_flag) {
        if (a_armed) drain_wait(bar(B_AF), (a_armed - 1) & 1u);
        // Stage s received ceil((issued - s) / N) loads; wait for the last.
        for (uint32_t s = 0; s < NX; ++s) {
          const uint32_t nx = (x_issued + NX - 1 - s) / NX;
          if (nx) drain_wait(bar(B_XF + s), (nx - 1) & 1u);
        }
        for (uint32_t s = 0; s < NY; ++s) {
          const uint32_t ny = (y_issued + NY - 1 - s) / NY;
          if (ny) drain_wait(bar(B_YF + s), (ny - 1) & 1u);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == 2) {
    // ---------------------------------------------------- MMA issuers ----
    // Each issuer is a whole warp in uniform control flow; one elected lane
    // issues its MMAs and commits (faster issue than a lone lane while the
    // softmax warps share the scheduler).
    {
      const bool issuer_a = warp == 1;
      auto wait_w = [&](uint32_t b_, uint32_t par_) -> bool {
        return __all_sync(0xffffffffu, wait_bar(b_, par_, p, abort_flag));
      };
      const uint64_t a0_desc = sdesc_sw128(base + LY::A0, 16, 1024);
      const uint64_t a1_desc = sdesc_sw128(base + LY::A1, 16, 1024);
      const uint64_t xk_desc = sdesc_sw128(base + LY::X, 16, 1024);       // K-major view
      const uint64_t xm_desc = sdesc_sw128(base + LY::X, kTH, 1024);      // MN-major view
      const uint64_t yk_desc = sdesc_sw128(base + LY::Y, 16, 1024);
      const uint64_t ym_desc = sdesc_sw128(base + LY::Y, kTH, 1024);
      // First MMAs of tile t: S = A0 X^T (issuer A) or dP = A1 Y^T (issuer B).
      // ready: the stage barrier was already seen complete (a test this
      // thread ran during its previous accumulating MMAs).
      // bs: the S/dP buffer of c.t (index and use parity).
      auto issue_first = [&](const Cursor& c, bool s_mma, const Stage& st, const Stage& bs,
                             bool ready) -> bool {
        const uint32_t b = bs.s;
        if (c.j == 0 && !wait_w(bar(B_AF), c.item_idx & 1)) return false;
        uint32_t stage;
        uint64_t bdesc;
        if (s_mma) {
          // S part b (dQ pass) or buffer b's S^T part (dK/dV pass) last held
          // tile t-2; issuer A issued acc(t-2), which reads it, before this
          // in its own order.
          stage = st.s;
          if (!__all_sync(0xffffffffu, ready) && !wait_w(bar(B_XF + stage), st.ph)) return false;
          bdesc = xk_desc + stage * (kTL >> 4);
        } else {
          // dP(t) overwrites a dP part. dQ pass: the one dP part, once the
          // softmax warps have loaded dP(t-1) from it (dS goes to the S
          // part). dK/dV pass: gK(t-2), which reads dS^T from buffer b's dP
          // part, was issued by this thread first.
          if (!kKV && c.t >= 1 && !wait_w(bar(B_DR), (c.t - 1) & 1u)) return false;
          stage = st.s;
          if (!__all_sync(0xffffffffu, ready) && !wait_w(bar(B_YF + stage), st.ph)) return false;
          bdesc = yk_desc + stage * (kTL >> 4);
        }
        tc_fence_after();
        const uint32_t d = tmem + (s_mma ? s_col<kKV>(b) : dp_col<kKV>(b));
        // k-steps 4h .. 4h+3 (head-dim columns [64 h, 64 h + 64), one
        // swizzled half of each operand), four MMAs per elect.
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          const uint64_t bh = bdesc + ((h * kTH) >> 4);
          const uint64_t ah = (s_mma ? a0_desc : a1_desc) + ((h * kRHalf) >> 4);
          mma_ss4_elect(d, ah, ah + 2, ah + 4, ah + 6, bh, bh + 2, bh + 4, bh + 6, kIdescFirst<kKV>,
                        h > 0);
        }
        mma_commit_elect(bar(B_SF + b));
        if (!s_mma && !kKV) mma_commit_elect(bar(B_YE + stage));  // dQ pass: V feeds dP only
        if (c.j == c.n - 1) mma_commit_elect(bar(B_AE));   // done with A0 (S) / A1 (dP)
        return true;
      };
      // Accumulating MMAs. The bf16 operands of a tile sit at the start of
      // each 32-column step of S columns the softmax warps read (k-step ks at
      // column 32 (ks >> 1) + 8 (ks & 1)) in the S part (dQ pass: dS; dK/dV
      // pass: P^T) and, dK/dV pass, in the dP part (dS^T). dQ pass: gQ += dS
      // K, issuer A. dK/dV pass: gV += P^T G by issuer A (it reads the S
      // part), gK += dS^T Q by issuer B (the dP part), each followed in its
      // own thread by the first MMA that overwrites that part two tiles
      // later.
      // next_bar / next_ph: the stage barrier of this issuer's next first
      // MMAs (0: none). It is tested here, before this tile's MMAs are
      // issued, and the result is used only after them, so the test's
      // latency overlaps the issue. A completed phase stays complete until
      // this thread has issued the MMAs that read the stage, and every
      // earlier use of the stage completed under this thread's own waits.
      auto issue_acc = [&](const Cursor& c, bool s_part, const Stage& st, const Stage& bs,
                           uint32_t next_bar, uint32_t next_ph, bool& next_ready) -> bool {
        // X stage of tile t; in the dK/dV pass (NX == NY) also its Y stage.
        const uint32_t b = bs.s, sx = st.s, sy = st.s;
        if (c.j == 0 && c.item_idx > 0 &&
            !wait_w(bar(B_CF), (c.item_idx - 1) & 1))
          return false;
        if (!wait_w(bar(B_PF + b), bs.ph)) return false;
        next_ready = next_bar != 0u && mbar_test(next_bar, next_ph);
        tc_fence_after();
        const uint32_t first = c.j == 0 ? 0u : 1u;
        const uint32_t a_p = tmem + (s_part ? s_col<kKV>(b) : dp_col<kKV>(b));
        // B operand: dQ pass K (X); dK/dV pass G (Y) for gV, Q (X) for gK.
        const uint64_t bm = (!kKV || !s_part) ? xm_desc + sx * (kTL >> 4)
                                              : ym_desc + sy * (kTL >> 4);
        const uint32_t acc = (!kKV || s_part) ? kC0<kKV> : TM_C1;
        // k-step ks of 16 streamed rows: A columns 32 (ks >> 1) + 8 (ks & 1),
        // B rows 16 ks (eight steps in the dQ pass, four in the dK/dV pass).
        mma_ts4_elect(tmem + acc, a_p, a_p + 8u, a_p + 32u, a_p + 40u, bm, bm + 128, bm + 256,
                      bm + 384, IDESC_MN, first);
        if (!kKV)
          mma_ts4_elect(tmem + acc, a_p + 64u, a_p + 72u, a_p + 96u, a_p + 104u, bm + 512,
                        bm + 640, bm + 768, bm + 896, IDESC_MN, 1u);
        // Stage release: dQ pass, this thread read X(t) (also with S(t),
        // earlier) and Y(t) only through dP(t); dK/dV pass, both issuers
        // commit to the pair's one barrier (X and Y feed one MMA batch of
        // each: S^T and gK, dP^T and gV). At an item's last tile, the
        // accumulation-done the epilogue waits for.
        mma_commit_elect(bar(B_XE + sx));
        if (c.j == c.n - 1) mma_commit_elect(bar(B_MD));
        return true;
      };
      bool ok = true;
      if (issuer_a) {
        // acc(t), then S(t+2) in this thread's order: S(t+2) overwrites the
        // S part of the buffer acc(t) reads. S runs up to two tiles ahead of
        // acc but not into the next item, whose stationary operands are
        // loaded once both issuers are done with this item's.
        Cursor cs, ca;
        Stage ss, sa;    // X stages of cs.t and ca.t
        Stage bss, bsa;  // S/dP buffers of cs.t and ca.t
        cs.start(p, ring, kConsumerWarp);
        ca.start(p, ring, kConsumerWarp);
        // Failure-detection test: wait on the drain barrier's first phase,
        // which nothing completes before this warp's own drain commit, so the
        // bounded wait runs out and the abort path below is taken.
        if (p.stall_test) ok = __all_sync(0xffffffffu, wait_bar(bar(B_DRAIN + 0), 0u, p, abort_flag));
        bool xr = false;  // XF of cs.t seen complete
        while (ok && ca.valid) {
          while (ok && cs.valid && cs.t < ca.t + kBufs<kKV> && cs.item_idx == ca.item_idx) {
            ok = issue_first(cs, true, ss, bss, xr);
            xr = false;
            cs.next(p, ring, kConsumerWarp);
            ss.step(NX);
            bss.step(kBufs<kKV>);
          }
          if (!ok) break;
          ok = issue_acc(ca, true, sa, bsa, cs.valid ? bar(B_XF + ss.s) : 0u, ss.ph, xr);
          ca.next(p, ring, kConsumerWarp);
          sa.step(NX);
          bsa.step(kBufs<kKV>);
        }
      } else if (!kKV) {
        // dP of every tile, as soon as its buffer part is free.
        Cursor c;
        Stage sc, bsc;  // Y stage and S/dP buffer of c.t
        c.start(p, ring, kConsumerWarp);
        while (c.valid && ok) {
          ok = issue_first(c, false, sc, bsc, false);
          c.next(p, ring, kConsumerWarp);
          sc.step(NY);
          bsc.step(kBufs<kKV>);
        }
      } else {
        // gK(t), then dP^T(t+2) in this thread's order (it overwrites the dP
        // part gK(t) reads), as issuer A does with the S part.
        Cursor cd, ck;
        Stage sd, sk;    // stages (X and Y alike) of cd.t and ck.t
        Stage bsd, bsk;  // S/dP buffers of cd.t and ck.t
        cd.start(p, ring, kConsumerWarp);
        ck.start(p, ring, kConsumerWarp);
        bool yr = false;  // YF of cd.t seen complete
        while (ok && ck.valid) {
          while (ok && cd.valid && cd.t < ck.t + kBufs<kKV> && cd.item_idx == ck.item_idx) {
            ok = issue_first(cd, false, sd, bsd, yr);
            yr = false;
            cd.next(p, ring, kConsumerWarp);
            sd.step(NY);
            bsd.step(kBufs<kKV>);
          }
          if (!ok) break;
          ok = issue_acc(ck, false, sk, bsk, cd.valid ? bar(B_YF + sd.s) : 0u, sd.ph, yr);
          ck.next(p, ring, kConsumerWarp);
          sk.step(NX);
          bsk.step(kBufs<kKV>);
        }
      }
      if (__any_sync(0xffffffffu, !ok || *abort_flag)) {
        const uint32_t db = bar(B_DRAIN + (issuer_a ? 0 : 1));
        mma_commit_elect(db);
        drain_wait(db, 0);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------ softmax warps ----
    const int hw = (warp - 4) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t tl = tmem + (uint32_t(q4 * 32) << 16);
    const int chunk = p.mask.chunk < 1 ? 1 : p.mask.chunk;
    const float kLog2e = 1.4426950408889634f;
    Cursor c;
    Stage bsm;  // S/dP buffer of c.t
    c.start(p, ring, kConsumerWarp);
    RowKeys rk{0, 0, 0, 0};
    int grow = 0;
    // dQ pass: this row's LSE (log2, +inf past L so that P = 0 there) and D.
    float lse2 = 0.f, dval = 0.f;
    bool ok = true;
    while (c.valid) {
      if (c.j == 0) {
        grow = c.qt * BR + r;
        if (!kKV) {
          rk = row_keys(p.mask.mode, p.mask.tokens_per_frame, p.mask.n_frames, chunk, p.L, grow);
          lse2 = CUDART_INF_F;
          dval = 0.f;
          const size_t roff = size_t(c.bh) * p.L + grow;
          if (grow < p.L) {
            const float l = p.lse[roff];
            if (l != -CUDART_INF_F) lse2 = l * kLog2e;
            // D = <g, o> for this row, both 128-wide rows read as 16 B vectors.
            const uint4* gr = reinterpret_cast<const uint4*>(p.g + roff * D);
            const uint4* orow = reinterpret_cast<const uint4*>(p.o + roff * D);
            float acc = 0.f;
#pragma unroll 4
            for (int i = 0; i < D / 8; ++i) {
              const uint4 a = gr[i], bq = orow[i];
              const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
              const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&bq);
#pragma unroll
              for (int k2 = 0; k2 < 4; ++k2) {
                const float2 fa = __bfloat1622float2(a2[k2]), fb = __bfloat1622float2(b2[k2]);
                acc = fmaf(fa.x, fb.x, fmaf(fa.y, fb.y, acc));
              }
            }
            dval = acc;
          }
          // grow < Lp always: the last query tile covers the padding rows.
          if (hw == 0) {
            float* sdp = p.sd + (size_t(c.bh) * p.Lp + (grow & ~1)) * 2 + (grow & 1);
            sdp[0] = -lse2;
            sdp[2] = -dval;
          }
        } else {
          rk = key_queries(p.mask.mode, p.mask.tokens_per_frame, p.mask.n_frames, chunk, p.L,
                           grow);
        }
      }
      // Column indices of this thread's 32 elements of a step: keys (dQ
      // pass: two steps, columns 64 hw + 32 h2 of the 128-key tile) or
      // queries (dK/dV pass: one step, columns 32 hw) [col0, col0 + 32).
      int col0 = c.kt * BT + 32 * hw;
      // dK/dV pass: -LSE2 and -D of this warpgroup's 32 queries, 16 query
      // pairs of {-LSE2 pair, -D pair} (two packed fp32 pairs each, the same
      // for every lane), read from the tile's shared-memory slice where they
      // are used.
      const ulonglong2* wsrc = nullptr;
      if (kKV) {
        // The slice arrived with the tile's Q stage; that stage's barrier is
        // still in this tile's phase (the stage is reloaded only after this
        // tile's accumulating MMAs, which wait for these warps).
        const uint32_t sx = c.t % NX;
        ok = wait_bar(bar(B_XF + sx), (c.t / NX) & 1u, p, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) break;
        wsrc = reinterpret_cast<const ulonglong2*>(base_ptr + LY::W + sx * 512u) + 16 * hw;
      }
      const uint32_t b = bsm.s;
      ok = wait_bar(bar(B_SF + b), bsm.ph, p, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t sr[32] = {}, dr[32] = {};
      uint32_t pp[16], pd[16];
      // Elements (2i, 2i+1) as one packed fp32 pair: P = 2^(c2 S - LSE2),
      // dS = P (dP - D), each rounded as the scalar expression would be;
      // zero where the mask excludes the pair (only partial tiles test it).
      const uint64_t c2v = f2pack(p.c2, p.c2);
      const uint64_t nl_row = f2pack(-lse2, -lse2), nd_row = f2pack(-dval, -dval);  // dQ pass
      auto pair = [&](int i, bool masked) {
        ulonglong2 wv = make_ulonglong2(nl_row, nd_row);
        if (kKV) wv = wsrc[i];
        const uint64_t nl = wv.x, nd = wv.y;
        float x0, x1, e0, e1, d0, d1;
        f2unpack(fma2(f2pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), c2v, nl),
                 x0, x1);
        e0 = ex2(x0);
        e1 = ex2(x1);
        const uint64_t dsv =
            mul2(f2pack(e0, e1),
                 add2(f2pack(__uint_as_float(dr[2 * i]), __uint_as_float(dr[2 * i + 1])), nd));
        f2unpack(dsv, d0, d1);
        if (masked) {
          if (!key_ok(rk, col0 + 2 * i)) e0 = d0 = 0.f;
          if (!key_ok(rk, col0 + 2 * i + 1)) e1 = d1 = 0.f;
        }
        pp[i] = pack_bf16(e0, e1);
        pd[i] = pack_bf16(d0, d1);
      };
      auto step = [&]() {
        if (c.partial) {
#pragma unroll
          for (int i = 0; i < 16; ++i) pair(i, true);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) pair(i, false);
        }
      };
      if (!kKV) {
        // dQ pass: warpgroup hw takes keys [64 hw, 64 hw + 64) of the tile in
        // two steps of 32; dS goes back over the start of each step's S
        // columns (packed column 32 (ks >> 1) + 8 (ks & 1) for k-step ks).
        // Both steps' dP are loaded up front, so the dP part is released
        // before any arithmetic, and the second step's S load is in flight
        // while the first step's dS is stored.
        {
          const uint32_t col = 64u * hw;
          uint32_t dr1[32];
          tmem_ld32(tl + s_col<kKV>(b) + col, sr);
          tmem_ld32(tl + dp_col<kKV>(b) + col, dr);
          tmem_ld32(tl + dp_col<kKV>(b) + col + 32u, dr1);
          tmem_wait_ld();
          // Both steps' dP are in registers: the dP part may take the next tile's dP.
          tc_fence_before();
          mbar_arrive(bar(B_DR));
          col0 = c.kt * BT + int(col);
          step();
          tmem_st16(tl + s_col<kKV>(b) + col, pd);
          tmem_ld32(tl + s_col<kKV>(b) + col + 32u, sr);
#pragma unroll
          for (int i = 0; i < 32; ++i) dr[i] = dr1[i];
          tmem_wait_ld();
          col0 = c.kt * BT + int(col) + 32;
          step();
          tmem_st16(tl + s_col<kKV>(b) + col + 32u, pd);
        }
      } else {
        tmem_ld32(tl + s_col<kKV>(b) + 32u * hw, sr);
        tmem_ld32(tl + dp_col<kKV>(b) + 32u * hw, dr);
        tmem_wait_ld();
        step();
        tmem_st16(tl + s_col<kKV>(b) + 32u * hw, pp);   // P^T over its S^T columns
        tmem_st16(tl + dp_col<kKV>(b) + 32u * hw, pd);  // dS^T over its dP^T columns
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_PF + b));

      if (c.j == c.n - 1) {
        // ------------------------------------------------------ epilogue --
        // The previous phase of this barrier (the previous item's) is the
        // one this warp waited for in that item's epilogue; the next cannot
        // complete before this epilogue arrives on B_CF.
        ok = wait_bar(bar(B_MD), c.item_idx & 1, p, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
        const bool row_ok = grow < p.L;
        const size_t off = (size_t(c.bh) * p.L + (row_ok ? grow : 0)) * D;
        // Warpgroup hw writes head-dim columns [64 hw, 64 hw + 64) of each output.
#pragma unroll 1
        for (int oi = 0; oi < (kKV ? 2 : 1); ++oi) {
          // dQ pass: gQ = c * C0. dK/dV pass: gK = c * C1, gV = C0.
          const uint32_t acc_col = !kKV ? kC0<kKV> : (oi == 0 ? TM_C1 : kC0<kKV>);
          const float mul = (!kKV || oi == 0) ? p.scale : 1.f;
          __nv_bfloat16* dst = (!kKV || oi == 0) ? p.out0 : p.out1;
#pragma unroll 1
          for (int cc = 0; cc < 2; ++cc) {
            const uint32_t col = 64u * hw + 32u * cc;
            uint32_t a[32];
            tmem_ld32(tl + acc_col + col, a);
            tmem_wait_ld();
            uint32_t po[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              po[i] = pack_bf16(__uint_as_float(a[2 * i]) * mul,
                                __uint_as_float(a[2 * i + 1]) * mul);
            if (row_ok) {
              uint4* go = reinterpret_cast<uint4*>(dst + off + col);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                go[i] = make_uint4(po[4 * i], po[4 * i + 1], po[4 * i + 2], po[4 * i + 3]);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(bar(B_CF));
      }
      c.next(p, ring, kConsumerWarp);
      bsm.step(kBufs<kKV>);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
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

static bool make_map(CUtensorMap* m, const void* ptr, int L, int BH, int rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(L), cuuint64_t(BH)};
  cuuint64_t strides[2] = {cuuint64_t(D) * 2, cuuint64_t(L) * D * 2};
  cuuint32_t box[3] = {64, cuuint32_t(rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kKV>
static int launch_pass(const BwdArgs& a, const WorkList& w, int num_sms, unsigned* ctr) {
  const int BH = a.B * a.H;
  CUtensorMap m0, m1, mx, my;
  // dQ pass: stationary Q, G; streamed K, V.  dK/dV: stationary K, V; streamed Q, G.
  const void* s0 = kKV ? a.k : a.q;
  const void* s1 = kKV ? a.v : a.g;
  const void* sx = kKV ? a.q : a.k;
  const void* sy = kKV ? a.g : a.v;
  if (!make_map(&m0, s0, a.L, BH, BR) || !make_map(&m1, s1, a.L, BH, BR) ||
      !make_map(&mx, sx, a.L, BH, kBT<kKV>) || !make_map(&my, sy, a.L, BH, kBT<kKV>))
    return JVP_ERR_LAUNCH_FAILED;
  Params p;
  p.qtiles = w.qtiles;
  p.segs = w.segs;
  p.n_entries = w.n_qtiles;
  p.n_segs = w.n_segs;
  const long long items = (long long)w.n_qtiles * BH;
  if (items > 0x7fffffffLL) return JVP_ERR_TOO_LARGE;
  p.n_items = int(items);
  p.n_qt = (a.L + BR - 1) / BR;
  p.n_kt = (a.L + kBT<kKV> - 1) / kBT<kKV>;
  p.L = a.L;
  p.mask = a.mask;
  p.scale = a.scale;
  p.c2 = a.scale * 1.4426950408889634f;
  p.lse = a.lse;
  p.Lp = (a.L + 127) / 128 * 128;
  p.sd = a.scratch;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.g = static_cast<const __nv_bfloat16*>(a.g);
  p.o = static_cast<const __nv_bfloat16*>(a.o);
  p.out0 = static_cast<__nv_bfloat16*>(kKV ? a.gk : a.gq);
  p.out1 = static_cast<__nv_bfloat16*>(a.gv);
  p.err = a.err;
  p.item_ctr = ctr;
  p.wait_limit_ns = a.wait_limit_ns;
  p.stall_test = a.stall_test ? 1 : 0;
  static std::mutex attr_mu;
  static bool attr_done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return JVP_ERR_LAUNCH_FAILED;
  {
    std::lock_guard<std::mutex> lk(attr_mu);
    if (!attr_done[dev]) {
      if (cudaFuncSetAttribute(bwd_kernel<kKV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Layout<kKV>::kBytes) != cudaSuccess)
        return JVP_ERR_LAUNCH_FAILED;
      attr_done[dev] = true;
    }
  }
  const int grid = int(items < num_sms ? items : num_sms);
  if (cudaMemsetAsync(ctr, 0, sizeof(unsigned), a.stream) != cudaSuccess)
    return JVP_ERR_LAUNCH_FAILED;
  bwd_kernel<kKV><<<grid, kThreads, Layout<kKV>::kBytes, a.stream>>>(m0, m1, mx, my, p);
  return cudaGetLastError() == cudaSuccess ? JVP_OK : JVP_ERR_LAUNCH_FAILED;
}

}  // namespace bwd

int launch_bwd_sm100(const BwdArgs& a, const WorkList& wq, const WorkList& wkv, int num_sms) {
  if (!a.item_ctr) return JVP_ERR_LAUNCH_FAILED;
  int rc = bwd::launch_pass<false>(a, wq, num_sms, a.item_ctr);
  if (rc != JVP_OK) return rc;
  // The second pass reads D from the first one (stream-ordered) and uses the
  // second counter word.
  return bwd::launch_pass<true>(a, wkv, num_sms, a.item_ctr + 1);
}

}  // namespace jvp
