// Internal declarations shared by the C-ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/jvp_attn.h"

namespace jvp {

// Bits of the per-device error word the kernels OR into.
constexpr unsigned kErrTimeout = 1u;
constexpr unsigned kErrBounds = 2u;

// Device work list for the tensor-core kernel (see schedule.h).
struct WorkList {
  const int4* qtiles = nullptr;  // {qt, seg_begin, seg_count, n_ktiles}
  const int2* segs = nullptr;    // {kt_begin, (count << 1) | partial}
  int n_qtiles = 0;
  int n_segs = 0;
};

// Destinations of the scatter epilogue (token shards of a Ulysses group).
constexpr int kMaxShards = 8;

struct LaunchArgs {
  const void *q, *k, *v, *dq, *dk, *dv;
  void *o, *d_o;
  float* lse;
  int B, H, L, d;
  jvp_mask_desc mask;
  float scale;
  cudaStream_t stream;
  unsigned* err;  // device error word
  // Work-item counter of the tensor-core kernel (one u32 of device memory
  // owned by the caller of launch_sm100, which zeroes it on `stream` before
  // the launch). Launches that share a counter must be stream-ordered.
  unsigned* item_ctr = nullptr;
  unsigned long long wait_limit_ns;
  bool stall_test = false;  // jvp_attn_set_stall_test
  // Scatter epilogue (jvp_attn_fwd_scatter), tensor-core kernel only: when
  // n_shards > 0, o / d_o / lse are unused and row n of local head (b, h)
  // goes to token-shard owner r = n / (L / n_shards), row n % (L / n_shards)
  // of head h0 + h in o_dst[r], d_o_dst[r], lse_dst[r] ([B, h_total, L/n_shards, d]).
  int n_shards = 0, h0 = 0, h_total = 0;
  void* o_dst[kMaxShards] = {};
  void* d_o_dst[kMaxShards] = {};
  float* lse_dst[kMaxShards] = {};
};

// CUDA-core kernel (fp32 arithmetic) for fp32 or bf16 inputs, d in {32,64,96,128}.
int launch_simt(const LaunchArgs& a, bool bf16);

// Tensor-core kernel: bf16, d = 128, sm_100a.
int launch_sm100(const LaunchArgs& a, const WorkList& w, int num_sms);

struct BwdArgs {
  const void *q, *k, *v, *o, *g;  // g: cotangent of o
  const float* lse;               // forward LSE
  void *gq, *gk, *gv;
  float* scratch;                 // [B*H, Lp, 2]: per row pair, -LSE*log2(e) of both
                                  // rows then -D = -<g, o> of both; Lp = L rounded
                                  // up to a multiple of 128
  int B, H, L, d;
  jvp_mask_desc mask;
  float scale;
  cudaStream_t stream;
  unsigned* err;
  unsigned* item_ctr;  // two u32 words: one per pass
  unsigned long long wait_limit_ns;
  bool stall_test = false;  // jvp_attn_set_stall_test
};

// Backward passes (dQ, then dK/dV): bf16, d = 128, sm_100a. wq: query-tile
// work list (128 x 64 grid); wkv: key-tile work list (64 x 128 grid).
int launch_bwd_sm100(const BwdArgs& a, const WorkList& wq, const WorkList& wkv, int num_sms);

// Chunk attention over a key/value cache (jvp_attn_cache_fwd): bf16, d = 128.
struct CacheArgs {
  const void *q, *k, *v;  // q [B, H, Lq, d]; k, v caches [B, H, Lcache, d]
  void* o;                // [B, H, Lq, d]
  float* lse;             // [B, H, Lq]
  int B, H, Lq, Lk, Lcache;
  float scale;
  cudaStream_t stream;
  unsigned* err;
  unsigned* item_ctr;
  unsigned long long wait_limit_ns;
  bool stall_test = false;  // jvp_attn_set_stall_test
  float* part;  // [slots, 128, 128] fp32 partial outputs (pieces of split items)
  float* ml;    // [slots, 128] {max, sum} pairs
};

// Device copy of a cache-attention work list (build_schedule_cache, 128 x
// 128 tiles): the pieces as a WorkList plus their {bh, slot}, and the cut
// items {bh, qt, first slot, slot count}.
struct CacheWork {
  WorkList w;
  const int2* meta = nullptr;
  const int4* splits = nullptr;
  int n_splits = 0, n_slots = 0;
};

int launch_cache_sm100(const CacheArgs& a, const CacheWork& cw, int num_sms);

// Row copy with optional rotary embedding (jvp_attn_rope_copy).
struct RopeArgs {
  const void* src;
  void* dst;
  int B, H, src_rows, dst_rows, rows, src_row0, dst_row0, d;
  bool bf16;
  const float *cos, *sin;  // both null: plain copy
  int rope_row0;
  cudaStream_t stream;
};
int launch_rope_copy(const RopeArgs& a, int num_sms);

// Device-side barrier of n <= kMaxShards ranks (jvp_attn_signal_barrier).
int launch_signal_barrier(uint32_t* const* flags, int n, int rank, uint32_t epoch,
                          unsigned* err, unsigned long long limit_ns, cudaStream_t st);

// Attention-layer tangent prologue (jvp_attn_qkv_prologue): bf16.
struct PrologueArgs {
  const void *qkv, *dqkv;  // [B, L, 3 H d]
  void* out[6];            // q, k, v, dq, dk, dv: [B, H, L, d]
  const float *norm_q, *norm_k;  // [group] or null (no norm)
  const float *cos, *sin;        // [>= L, d/2] or null (no rotation)
  int B, L, H, d, group;
  float eps;
  cudaStream_t stream;
};
int launch_qkv_prologue(const PrologueArgs& a, int num_sms);

// Per-wait limit for the tensor-core kernels (jvp_attn_set_wait_limit).
unsigned long long wait_limit_ns();
// Failure-detection test switch of the tensor-core kernels (jvp_attn_set_stall_test).
bool stall_test();

// Current device's SM count and error word; JVP_ERR_UNSUPPORTED_DEVICE
// unless it is an sm_100 device. Allocates nothing.
int current_device_state(int* sms, unsigned** err);

}  // namespace jvp
