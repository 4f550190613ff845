// C ABI of the masked attention JVP library (declared in include/jvp_attn.h).
//
// Host-side duties: argument validation, the per-device error word, the
// cached device work lists built by the tile scheduler, and dispatch to the
// tensor-core kernel (bf16, d = 128) or the CUDA-core kernel (fp32 / other
// head dims). No exception crosses the boundary.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "common.cuh"
#include "schedule.h"

// One error word per device that loads the library; kernels OR bits in.
__device__ unsigned g_jvp_error_word;

namespace jvp {
namespace {

constexpr int kBM = 128, kBN = 64;            // tensor-core tile shape
constexpr unsigned long long kDefaultWaitLimitNs = 2000000000ull;  // 2 s per wait
std::atomic<unsigned long long> g_wait_limit{kDefaultWaitLimitNs};
std::atomic<bool> g_stall_test{false};
constexpr int kMaxDevices = 64;

struct DevInfo {
  bool ready = false;
  int sms = 0, major = 0, minor = 0;
  unsigned* err = nullptr;
};

struct WsKey {
  // kind 0: query-tile list, 1: key-tile list (mask fields), 3: cache
  // attention list (T = grid, F = B*H, chunk = Lq, L = Lk).
  int dev, mode, T, F, chunk, L, bm, bn, kind;
  bool operator<(const WsKey& o) const {
    return std::tie(dev, mode, T, F, chunk, L, bm, bn, kind) <
           std::tie(o.dev, o.mode, o.T, o.F, o.chunk, o.L, o.bm, o.bn, o.kind);
  }
};

struct Ws {
  void* buf = nullptr;
  WorkList w;
  CacheWork cw;  // kind 3 only
};

std::mutex g_mu;
DevInfo g_dev[kMaxDevices];
std::map<WsKey, Ws> g_ws;
// Work-item counter of the tensor-core kernel, one per (device, stream):
// launches on one stream are ordered, so they can share it.
std::map<std::pair<int, cudaStream_t>, unsigned*> g_ctr;
// Split-K partial results of cache attention, per (device, stream), grown
// on demand: {buffer, bytes}.
std::map<std::pair<int, cudaStream_t>, std::pair<void*, size_t>> g_part;

int device_info(DevInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return JVP_ERR_LAUNCH_FAILED;
  if (dev < 0 || dev >= kMaxDevices) return JVP_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  DevInfo& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) !=
            cudaSuccess)
      return JVP_ERR_LAUNCH_FAILED;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_jvp_error_word) != cudaSuccess) {
      cudaGetLastError();
      return JVP_ERR_UNSUPPORTED_DEVICE;  // no sm_100a image for this device
    }
    d.err = static_cast<unsigned*>(p);
    if (cudaMemset(d.err, 0, sizeof(unsigned)) != cudaSuccess) return JVP_ERR_LAUNCH_FAILED;
    d.ready = true;
  }
  *out = &d;
  return JVP_OK;
}

// Copies a host schedule into a new device buffer and caches it under key.
// Caller holds g_mu.
int upload_schedule(const WsKey& key, const Schedule& s, WorkList* out) {
  const size_t qbytes = s.qtiles.size() * sizeof(int32_t);
  const size_t sbytes = s.segs.size() * sizeof(int32_t);
  const size_t soff = (qbytes + 255) & ~size_t(255);
  Ws ws;
  if (cudaMalloc(&ws.buf, soff + sbytes) != cudaSuccess) {
    cudaGetLastError();
    return JVP_ERR_OUT_OF_MEMORY;
  }
  char* b = static_cast<char*>(ws.buf);
  if (cudaMemcpy(b, s.qtiles.data(), qbytes, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(b + soff, s.segs.data(), sbytes, cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaFree(ws.buf);
    return JVP_ERR_LAUNCH_FAILED;
  }
  ws.w.qtiles = reinterpret_cast<const int4*>(b);
  ws.w.segs = reinterpret_cast<const int2*>(b + soff);
  ws.w.n_qtiles = int(s.qtiles.size() / 4);
  ws.w.n_segs = int(s.segs.size() / 2);
  g_ws[key] = ws;
  *out = ws.w;
  return JVP_OK;
}

int get_worklist(int dev, const jvp_mask_desc& m, int L, WorkList* out, int bm = kBM,
                 int bn = kBN, int kind = 0) {
  const WsKey key{dev, m.mode, m.tokens_per_frame, m.n_frames,
                  m.chunk, L, bm, bn, kind};
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_ws.find(key);
  if (it != g_ws.end()) {
    *out = it->second.w;
    return JVP_OK;
  }
  const Schedule s = kind == 0 ? build_schedule(m, L, bm, bn) : build_schedule_kv(m, L, bm, bn);
  return upload_schedule(key, s, out);
}

// Work list of cache attention for (Lq, Lk, B*H) on `grid` CTAs, uploaded
// once and cached.
int get_worklist_cache(int dev, int Lq, int Lk, int BH, int grid, CacheWork* out) {
  const WsKey key{dev, -1, grid, BH, Lq, Lk, 128, 128, 3};
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_ws.find(key);
  if (it != g_ws.end()) {
    *out = it->second.cw;
    return JVP_OK;
  }
  const CacheSchedule s = build_schedule_cache(Lq, Lk, 128, 128, BH, grid);
  const std::vector<int32_t>* parts[] = {&s.entries, &s.segs, &s.meta, &s.splits};
  size_t off[5] = {0};
  for (int i = 0; i < 4; ++i)
    off[i + 1] = (off[i] + parts[i]->size() * sizeof(int32_t) + 255) & ~size_t(255);
  Ws ws;
  if (cudaMalloc(&ws.buf, off[4] + 256) != cudaSuccess) {
    cudaGetLastError();
    return JVP_ERR_OUT_OF_MEMORY;
  }
  char* b = static_cast<char*>(ws.buf);
  for (int i = 0; i < 4; ++i) {
    if (parts[i]->empty()) continue;
    if (cudaMemcpy(b + off[i], parts[i]->data(), parts[i]->size() * sizeof(int32_t),
                   cudaMemcpyHostToDevice) != cudaSuccess) {
      cudaFree(ws.buf);
      return JVP_ERR_LAUNCH_FAILED;
    }
  }
  CacheWork& cw = ws.cw;
  cw.w.qtiles = reinterpret_cast<const int4*>(b + off[0]);
  cw.w.segs = reinterpret_cast<const int2*>(b + off[1]);
  cw.w.n_qtiles = int(s.entries.size() / 4);
  cw.w.n_segs = int(s.segs.size() / 2);
  cw.meta = reinterpret_cast<const int2*>(b + off[2]);
  cw.splits = reinterpret_cast<const int4*>(b + off[3]);
  cw.n_splits = int(s.splits.size() / 4);
  cw.n_slots = s.n_slots;
  ws.w = cw.w;
  g_ws[key] = ws;
  *out = cw;
  return JVP_OK;
}

// Partial-result workspace of at least `bytes` for (dev, st).
int get_partials(int dev, cudaStream_t st, size_t bytes, void** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  auto& e = g_part[std::make_pair(dev, st)];
  if (e.first && e.second >= bytes) {
    *out = e.first;
    return JVP_OK;
  }
  if (e.first) {
    // Earlier launches on this stream may still read the old buffer.
    if (cudaStreamSynchronize(st) != cudaSuccess || cudaFree(e.first) != cudaSuccess)
      return JVP_ERR_LAUNCH_FAILED;
    e.first = nullptr;
    e.second = 0;
  }
  if (cudaMalloc(&e.first, bytes) != cudaSuccess) {
    cudaGetLastError();
    e.first = nullptr;
    return JVP_ERR_OUT_OF_MEMORY;
  }
  e.second = bytes;
  *out = e.first;
  return JVP_OK;
}

int get_counter(int dev, cudaStream_t st, unsigned** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  const auto key = std::make_pair(dev, st);
  auto it = g_ctr.find(key);
  if (it != g_ctr.end()) {
    *out = it->second;
    return JVP_OK;
  }
  void* p = nullptr;
  if (cudaMalloc(&p, 256) != cudaSuccess) {
    cudaGetLastError();
    return JVP_ERR_OUT_OF_MEMORY;
  }
  g_ctr[key] = static_cast<unsigned*>(p);
  *out = static_cast<unsigned*>(p);
  return JVP_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

unsigned long long wait_limit_ns() { return g_wait_limit.load(); }
bool stall_test() { return g_stall_test.load(); }

int current_device_state(int* sms, unsigned** err) {
  DevInfo* di = nullptr;
  const int rc = device_info(&di);
  if (rc != JVP_OK) return rc;
  if (di->major != 10 || di->minor != 0) return JVP_ERR_UNSUPPORTED_DEVICE;
  *sms = di->sms;
  *err = di->err;
  return JVP_OK;
}

}  // namespace jvp

using namespace jvp;

extern "C" {

int jvp_attn_fwd(const void* q, const void* k, const void* v, const void* dq, const void* dk,
                 const void* dv, void* o, void* d_o, float* lse, int B, int H, int L, int d,
                 jvp_dtype dtype, jvp_mask_desc mask, float softmax_scale, void* stream) {
  if (!q || !k || !v || !dq || !dk || !dv || !o || !d_o || !lse) return JVP_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || L <= 0 || d <= 0) return JVP_ERR_INVALID_ARG;
  if (dtype != JVP_BF16 && dtype != JVP_FP32) return JVP_ERR_INVALID_ARG;
  if (std::isnan(softmax_scale) || std::isinf(softmax_scale)) return JVP_ERR_INVALID_ARG;
  int rc = validate_mask(mask, L);
  if (rc != JVP_OK) return rc;
  if ((long long)B * H * L >= (1LL << 31) || (long long)B * H >= (1LL << 31) / 2)
    return JVP_ERR_TOO_LARGE;
  const bool tensor_core = dtype == JVP_BF16 && d == 128;
  if (!tensor_core && (d % 32 != 0 || d > 128)) return JVP_ERR_UNSUPPORTED_HEAD_DIM;
  const void* ptrs[] = {q, k, v, dq, dk, dv, o, d_o, lse};
  for (const void* p : ptrs)
    if (!aligned16(p)) return JVP_ERR_MISALIGNED;

  DevInfo* di = nullptr;
  rc = device_info(&di);
  if (rc != JVP_OK) return rc;
  if (di->major != 10 || di->minor != 0) return JVP_ERR_UNSUPPORTED_DEVICE;

  LaunchArgs a;
  a.q = q; a.k = k; a.v = v; a.dq = dq; a.dk = dk; a.dv = dv;
  a.o = o; a.d_o = d_o; a.lse = lse;
  a.B = B; a.H = H; a.L = L; a.d = d;
  a.mask = mask;
  a.scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(float(d));
  a.stream = static_cast<cudaStream_t>(stream);
  a.err = di->err;
  a.wait_limit_ns = wait_limit_ns();
  a.stall_test = stall_test();
  if (!tensor_core) return launch_simt(a, dtype == JVP_BF16);

  int dev = 0;
  cudaGetDevice(&dev);
  WorkList w;
  rc = get_worklist(dev, mask, L, &w);
  if (rc != JVP_OK) return rc;
  rc = get_counter(dev, a.stream, &a.item_ctr);
  if (rc != JVP_OK) return rc;
  return launch_sm100(a, w, di->sms);
}

int jvp_attn_fwd_scatter(const void* q, const void* k, const void* v, const void* dq,
                         const void* dk, const void* dv, void* const* o_dst,
                         void* const* d_o_dst, float* const* lse_dst, int n_shards, int h0,
                         int h_total, int B, int H, int L, int d, jvp_dtype dtype,
                         jvp_mask_desc mask, float softmax_scale, void* stream) {
  if (!q || !k || !v || !dq || !dk || !dv || !o_dst || !d_o_dst || !lse_dst)
    return JVP_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || L <= 0 || d <= 0) return JVP_ERR_INVALID_ARG;
  if (dtype != JVP_BF16 && dtype != JVP_FP32) return JVP_ERR_INVALID_ARG;
  if (std::isnan(softmax_scale) || std::isinf(softmax_scale)) return JVP_ERR_INVALID_ARG;
  if (n_shards < 1 || n_shards > kMaxShards || L % n_shards != 0) return JVP_ERR_INVALID_ARG;
  if (h0 < 0 || h_total < H || h0 > h_total - H) return JVP_ERR_INVALID_ARG;
  int rc = validate_mask(mask, L);
  if (rc != JVP_OK) return rc;
  if ((long long)B * h_total * L >= (1LL << 31) || (long long)B * H >= (1LL << 31) / 2)
    return JVP_ERR_TOO_LARGE;
  if (dtype != JVP_BF16 || d != 128) return JVP_ERR_UNSUPPORTED_HEAD_DIM;
  const void* ptrs[] = {q, k, v, dq, dk, dv};
  for (const void* p : ptrs)
    if (!aligned16(p)) return JVP_ERR_MISALIGNED;
  for (int r = 0; r < n_shards; ++r) {
    if (!o_dst[r] || !d_o_dst[r] || !lse_dst[r]) return JVP_ERR_INVALID_ARG;
    if (!aligned16(o_dst[r]) || !aligned16(d_o_dst[r]) || !aligned16(lse_dst[r]))
      return JVP_ERR_MISALIGNED;
  }

  DevInfo* di = nullptr;
  rc = device_info(&di);
  if (rc != JVP_OK) return rc;
  if (di->major != 10 || di->minor != 0) return JVP_ERR_UNSUPPORTED_DEVICE;

  LaunchArgs a;
  a.q = q; a.k = k; a.v = v; a.dq = dq; a.dk = dk; a.dv = dv;
  a.o = nullptr; a.d_o = nullptr; a.lse = nullptr;
  a.B = B; a.H = H; a.L = L; a.d = d;
  a.mask = mask;
  a.scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(float(d));
  a.stream = static_cast<cudaStream_t>(stream);
  a.err = di->err;
  a.wait_limit_ns = wait_limit_ns();
  a.stall_test = stall_test();
  a.n_shards = n_shards;
  a.h0 = h0;
  a.h_total = h_total;
  for (int r = 0; r < n_shards; ++r) {
    a.o_dst[r] = o_dst[r];
    a.d_o_dst[r] = d_o_dst[r];
    a.lse_dst[r] = lse_dst[r];
  }
  int dev = 0;
  cudaGetDevice(&dev);
  WorkList w;
  rc = get_worklist(dev, mask, L, &w);
  if (rc != JVP_OK) return rc;
  rc = get_counter(dev, a.stream, &a.item_ctr);
  if (rc != JVP_OK) return rc;
  return launch_sm100(a, w, di->sms);
}

int jvp_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* g_o,
                 const float* lse, void* g_q, void* g_k, void* g_v, float* scratch,
                 int64_t scratch_len, int B, int H, int L, int d, jvp_dtype dtype,
                 jvp_mask_desc mask, float softmax_scale, void* stream) {
  if (!q || !k || !v || !o || !g_o || !lse || !g_q || !g_k || !g_v || !scratch)
    return JVP_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || L <= 0 || d <= 0 || dtype != JVP_BF16) return JVP_ERR_INVALID_ARG;
  if (std::isnan(softmax_scale) || std::isinf(softmax_scale)) return JVP_ERR_INVALID_ARG;
  if (d != 128) return JVP_ERR_UNSUPPORTED_HEAD_DIM;
  int rc = validate_mask(mask, L);
  if (rc != JVP_OK) return rc;
  if ((long long)B * H * L >= (1LL << 31) || (long long)B * H >= (1LL << 31) / 2)
    return JVP_ERR_TOO_LARGE;
  if (scratch_len < jvp_attn_bwd_scratch_len(B, H, L)) return JVP_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, o, g_o, lse, g_q, g_k, g_v, scratch};
  for (const void* p : ptrs)
    if (!aligned16(p)) return JVP_ERR_MISALIGNED;
  DevInfo* di = nullptr;
  rc = device_info(&di);
  if (rc != JVP_OK) return rc;
  if (di->major != 10 || di->minor != 0) return JVP_ERR_UNSUPPORTED_DEVICE;
  int dev = 0;
  cudaGetDevice(&dev);
  BwdArgs a;
  a.q = q; a.k = k; a.v = v; a.o = o; a.g = g_o; a.lse = lse;
  a.gq = g_q; a.gk = g_k; a.gv = g_v; a.scratch = scratch;
  a.B = B; a.H = H; a.L = L; a.d = d;
  a.mask = mask;
  a.scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(float(d));
  a.stream = static_cast<cudaStream_t>(stream);
  a.err = di->err;
  a.wait_limit_ns = wait_limit_ns();
  a.stall_test = stall_test();
  WorkList wq, wkv;
  rc = get_worklist(dev, mask, L, &wq, 128, 128, 0);
  if (rc != JVP_OK) return rc;
  rc = get_worklist(dev, mask, L, &wkv, 64, 128, 1);
  if (rc != JVP_OK) return rc;
  rc = get_counter(dev, a.stream, &a.item_ctr);
  if (rc != JVP_OK) return rc;
  return launch_bwd_sm100(a, wq, wkv, di->sms);
}

int64_t jvp_attn_bwd_scratch_len(int B, int H, int L) {
  if (B <= 0 || H <= 0 || L <= 0) return -1;
  const int64_t Lp = (int64_t(L) + 127) / 128 * 128;
  return 2 * int64_t(B) * H * Lp;
}

int jvp_attn_cache_fwd(const void* q, const void* k_cache, const void* v_cache, void* o,
                       float* lse, int B, int H, int Lq, int Lk, int Lcache, int d,
                       jvp_dtype dtype, float softmax_scale, void* stream) {
  if (!q || !k_cache || !v_cache || !o || !lse) return JVP_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || Lq <= 0 || Lk <= 0 || Lcache < Lk || d <= 0 || dtype != JVP_BF16)
    return JVP_ERR_INVALID_ARG;
  if (std::isnan(softmax_scale) || std::isinf(softmax_scale)) return JVP_ERR_INVALID_ARG;
  if (d != 128) return JVP_ERR_UNSUPPORTED_HEAD_DIM;
  if ((long long)B * H * Lq >= (1LL << 31) || (long long)B * H * Lcache >= (1LL << 31))
    return JVP_ERR_TOO_LARGE;
  const void* ptrs[] = {q, k_cache, v_cache, o, lse};
  for (const void* p : ptrs)
    if (!aligned16(p)) return JVP_ERR_MISALIGNED;
  DevInfo* di = nullptr;
  int rc = device_info(&di);
  if (rc != JVP_OK) return rc;
  if (di->major != 10 || di->minor != 0) return JVP_ERR_UNSUPPORTED_DEVICE;
  int dev = 0;
  cudaGetDevice(&dev);
  CacheArgs a;
  a.q = q; a.k = k_cache; a.v = v_cache; a.o = o; a.lse = lse;
  a.B = B; a.H = H; a.Lq = Lq; a.Lk = Lk; a.Lcache = Lcache;
  a.scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(float(d));
  a.stream = static_cast<cudaStream_t>(stream);
  a.err = di->err;
  a.wait_limit_ns = wait_limit_ns();
  a.stall_test = stall_test();
  a.part = nullptr;
  a.ml = nullptr;
  CacheWork cw;
  rc = get_worklist_cache(dev, Lq, Lk, B * H, di->sms, &cw);
  if (rc != JVP_OK) return rc;
  if (cw.n_slots > 0) {
    const size_t part_bytes = size_t(cw.n_slots) * 128 * 128 * sizeof(float);
    void* buf = nullptr;
    rc = get_partials(dev, a.stream, part_bytes + size_t(cw.n_slots) * 128 * 2 * sizeof(float),
                      &buf);
    if (rc != JVP_OK) return rc;
    a.part = static_cast<float*>(buf);
    a.ml = reinterpret_cast<float*>(static_cast<char*>(buf) + part_bytes);
  }
  rc = get_counter(dev, a.stream, &a.item_ctr);
  if (rc != JVP_OK) return rc;
  return launch_cache_sm100(a, cw, di->sms);
}

int jvp_attn_rope_copy(const void* src, void* dst, int B, int H, int src_rows, int dst_rows,
                       int rows, int src_row0, int dst_row0, int d, jvp_dtype dtype,
                       const float* rope_cos, const float* rope_sin, int rope_rows,
                       int rope_row0, void* stream) {
  if (!src || !dst || B <= 0 || H <= 0 || d <= 0 || rows < 0 || src_row0 < 0 || dst_row0 < 0)
    return JVP_ERR_INVALID_ARG;
  if (dtype != JVP_BF16 && dtype != JVP_FP32) return JVP_ERR_INVALID_ARG;
  if (d % (dtype == JVP_BF16 ? 8 : 4) != 0) return JVP_ERR_INVALID_ARG;
  if ((long long)src_row0 + rows > src_rows || (long long)dst_row0 + rows > dst_rows)
    return JVP_ERR_INVALID_ARG;
  if ((rope_cos == nullptr) != (rope_sin == nullptr)) return JVP_ERR_INVALID_ARG;
  if (rope_cos && (rope_row0 < 0 || (long long)rope_row0 + rows > rope_rows))
    return JVP_ERR_INVALID_ARG;
  if ((long long)B * H * (src_rows > dst_rows ? src_rows : dst_rows) * d >= (1LL << 40))
    return JVP_ERR_TOO_LARGE;
  if (src == dst && src_row0 != dst_row0) return JVP_ERR_INVALID_ARG;
  if (!aligned16(src) || !aligned16(dst) || (rope_cos && (!aligned16(rope_cos) ||
                                                          !aligned16(rope_sin))))
    return JVP_ERR_MISALIGNED;
  if (rows == 0) return JVP_OK;
  DevInfo* di = nullptr;
  int rc = device_info(&di);
  if (rc != JVP_OK) return rc;
  if (di->major != 10 || di->minor != 0) return JVP_ERR_UNSUPPORTED_DEVICE;
  RopeArgs a;
  a.src = src; a.dst = dst; a.B = B; a.H = H;
  a.src_rows = src_rows; a.dst_rows = dst_rows; a.rows = rows;
  a.src_row0 = src_row0; a.dst_row0 = dst_row0; a.d = d;
  a.bf16 = dtype == JVP_BF16;
  a.cos = rope_cos; a.sin = rope_sin; a.rope_row0 = rope_row0;
  a.stream = static_cast<cudaStream_t>(stream);
  return launch_rope_copy(a, di->sms);
}

int jvp_attn_qkv_prologue(const void* qkv, const void* d_qkv, void* q, void* k, void* v,
                          void* dq, void* dk, void* dv, const float* norm_q,
                          const float* norm_k, int norm_group, float eps,
                          const float* rope_cos, const float* rope_sin, int rope_rows, int B,
                          int L, int H, int d, jvp_dtype dtype, void* stream) {
  const void* ptrs[] = {qkv, d_qkv, q, k, v, dq, dk, dv};
  for (const void* p : ptrs)
    if (!p) return JVP_ERR_INVALID_ARG;
  if (B <= 0 || L <= 0 || H <= 0 || d <= 0 || dtype != JVP_BF16) return JVP_ERR_INVALID_ARG;
  if (d < 8 || d > 256 || (d & (d - 1)) != 0) return JVP_ERR_UNSUPPORTED_HEAD_DIM;
  if ((H * d) % 256 != 0) return JVP_ERR_INVALID_ARG;
  if ((norm_q == nullptr) != (norm_k == nullptr)) return JVP_ERR_INVALID_ARG;
  if (norm_q && (norm_group != H * d && norm_group != d)) return JVP_ERR_INVALID_ARG;
  if (norm_q && (!(eps >= 0.f) || std::isinf(eps))) return JVP_ERR_INVALID_ARG;
  if ((rope_cos == nullptr) != (rope_sin == nullptr)) return JVP_ERR_INVALID_ARG;
  if (rope_cos && rope_rows < L) return JVP_ERR_INVALID_ARG;
  if ((long long)B * L * 3 * H * d >= (1LL << 40)) return JVP_ERR_TOO_LARGE;
  for (const void* p : ptrs)
    if (!aligned16(p)) return JVP_ERR_MISALIGNED;
  const void* opt[] = {norm_q, norm_k, rope_cos, rope_sin};
  for (const void* p : opt)
    if (p && !aligned16(p)) return JVP_ERR_MISALIGNED;
  DevInfo* di = nullptr;
  int rc = device_info(&di);
  if (rc != JVP_OK) return rc;
  if (di->major != 10 || di->minor != 0) return JVP_ERR_UNSUPPORTED_DEVICE;
  PrologueArgs a;
  a.qkv = qkv; a.dqkv = d_qkv;
  a.out[0] = q; a.out[1] = k; a.out[2] = v; a.out[3] = dq; a.out[4] = dk; a.out[5] = dv;
  a.norm_q = norm_q; a.norm_k = norm_k; a.cos = rope_cos; a.sin = rope_sin;
  a.B = B; a.L = L; a.H = H; a.d = d; a.group = norm_q ? norm_group : H * d; a.eps = eps;
  a.stream = static_cast<cudaStream_t>(stream);
  return launch_qkv_prologue(a, di->sms);
}

int jvp_attn_schedule_kv(jvp_mask_desc mask, int L, int bq, int bk, int32_t* ktiles,
                         int ktile_cap, int32_t* segs, int seg_cap, int* n_ktiles, int* n_segs) {
  int rc = validate_mask(mask, L);
  if (rc != JVP_OK) return rc;
  if (bq < 1 || bk < 1) return JVP_ERR_INVALID_ARG;
  const Schedule s = build_schedule_kv(mask, L, bq, bk);
  const int nk = int(s.qtiles.size() / 4), ns = int(s.segs.size() / 2);
  if (n_ktiles) *n_ktiles = nk;
  if (n_segs) *n_segs = ns;
  if (!ktiles || !segs || ktile_cap < nk || seg_cap < ns) return JVP_ERR_INVALID_ARG;
  std::memcpy(ktiles, s.qtiles.data(), s.qtiles.size() * sizeof(int32_t));
  for (int i = 0; i < ns; ++i) {
    segs[3 * i] = s.segs[2 * i];
    segs[3 * i + 1] = s.segs[2 * i + 1] >> 1;
    segs[3 * i + 2] = s.segs[2 * i + 1] & 1;
  }
  return JVP_OK;
}

int jvp_attn_mask_stats(jvp_mask_desc mask, int L, int bm, int bn, int64_t* pairs,
                        int64_t* full, int64_t* partial, int64_t* empty) {
  int rc = validate_mask(mask, L);
  if (rc != JVP_OK) return rc;
  if (bm < 1 || bn < 1) return JVP_ERR_INVALID_ARG;
  if (pairs) *pairs = count_pairs(mask, L);
  if (full || partial || empty) {
    const int n_qt = (L + bm - 1) / bm, n_kt = (L + bn - 1) / bn;
    std::vector<int8_t> row(n_kt);
    int64_t cnt[3] = {0, 0, 0};
    for (int qt = 0; qt < n_qt; ++qt) {
      classify_qtile(mask, L, bm, bn, qt, row.data());
      for (int8_t c : row) ++cnt[c];
    }
    if (full) *full = cnt[JVP_TILE_FULL];
    if (partial) *partial = cnt[JVP_TILE_PARTIAL];
    if (empty) *empty = cnt[JVP_TILE_EMPTY];
  }
  return JVP_OK;
}

int jvp_attn_tile_classes(jvp_mask_desc mask, int L, int bm, int bn, int8_t* out,
                          int64_t out_len) {
  int rc = validate_mask(mask, L);
  if (rc != JVP_OK) return rc;
  if (bm < 1 || bn < 1 || !out) return JVP_ERR_INVALID_ARG;
  const int n_qt = (L + bm - 1) / bm, n_kt = (L + bn - 1) / bn;
  if (out_len < (int64_t)n_qt * n_kt) return JVP_ERR_INVALID_ARG;
  for (int qt = 0; qt < n_qt; ++qt) classify_qtile(mask, L, bm, bn, qt, out + (int64_t)qt * n_kt);
  return JVP_OK;
}

int jvp_attn_schedule(jvp_mask_desc mask, int L, int bm, int bn, int32_t* qtiles, int qtile_cap,
                      int32_t* segs, int seg_cap, int* n_qtiles, int* n_segs) {
  int rc = validate_mask(mask, L);
  if (rc != JVP_OK) return rc;
  if (bm < 1 || bn < 1) return JVP_ERR_INVALID_ARG;
  const Schedule s = build_schedule(mask, L, bm, bn);
  const int nq = int(s.qtiles.size() / 4), ns = int(s.segs.size() / 2);
  if (n_qtiles) *n_qtiles = nq;
  if (n_segs) *n_segs = ns;
  if (!qtiles || !segs || qtile_cap < nq || seg_cap < ns) return JVP_ERR_INVALID_ARG;
  std::memcpy(qtiles, s.qtiles.data(), s.qtiles.size() * sizeof(int32_t));
  for (int i = 0; i < ns; ++i) {
    segs[3 * i] = s.segs[2 * i];
    segs[3 * i + 1] = s.segs[2 * i + 1] >> 1;
    segs[3 * i + 2] = s.segs[2 * i + 1] & 1;
  }
  return JVP_OK;
}

int jvp_attn_check_device_error(void* stream) {
  DevInfo* di = nullptr;
  int rc = device_info(&di);
  if (rc != JVP_OK) return rc;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return JVP_ERR_LAUNCH_FAILED;
  unsigned w = 0;
  if (cudaMemcpy(&w, di->err, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess)
    return JVP_ERR_LAUNCH_FAILED;
  if (w != 0 && cudaMemset(di->err, 0, sizeof(unsigned)) != cudaSuccess)
    return JVP_ERR_LAUNCH_FAILED;
  if (w & kErrTimeout) return JVP_ERR_DEVICE_TIMEOUT;
  if (w & kErrBounds) return JVP_ERR_DEVICE_BOUNDS;
  return JVP_OK;
}

int jvp_attn_signal_barrier(uint32_t* const* flags, int n_ranks, int rank, uint32_t epoch,
                            void* stream) {
  if (!flags || n_ranks < 1 || n_ranks > kMaxShards || rank < 0 || rank >= n_ranks)
    return JVP_ERR_INVALID_ARG;
  for (int q = 0; q < n_ranks; ++q) {
    if (!flags[q]) return JVP_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(flags[q]) & 3u) return JVP_ERR_MISALIGNED;
  }
  DevInfo* di = nullptr;
  const int rc = device_info(&di);
  if (rc != JVP_OK) return rc;
  if (di->major != 10 || di->minor != 0) return JVP_ERR_UNSUPPORTED_DEVICE;
  return launch_signal_barrier(flags, n_ranks, rank, epoch, di->err, wait_limit_ns(),
                               static_cast<cudaStream_t>(stream));
}

int jvp_attn_set_wait_limit(uint64_t ns) {
  g_wait_limit.store(ns == 0 ? kDefaultWaitLimitNs : (unsigned long long)ns);
  return JVP_OK;
}

int jvp_attn_set_stall_test(int enable) {
  g_stall_test.store(enable != 0);
  return JVP_OK;
}

int jvp_attn_release(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  int cur = 0;
  const bool have_dev = cudaGetDevice(&cur) == cudaSuccess;
  int rc = JVP_OK;
  for (auto& kv : g_ws) {
    if (cudaSetDevice(kv.first.dev) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess ||
        cudaFree(kv.second.buf) != cudaSuccess)
      rc = JVP_ERR_LAUNCH_FAILED;
  }
  g_ws.clear();
  for (auto& kv : g_ctr) {
    if (cudaSetDevice(kv.first.first) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess ||
        cudaFree(kv.second) != cudaSuccess)
      rc = JVP_ERR_LAUNCH_FAILED;
  }
  g_ctr.clear();
  for (auto& kv : g_part) {
    if (!kv.second.first) continue;
    if (cudaSetDevice(kv.first.first) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess ||
        cudaFree(kv.second.first) != cudaSuccess)
      rc = JVP_ERR_LAUNCH_FAILED;
  }
  g_part.clear();
  if (have_dev) cudaSetDevice(cur);
  return rc;
}

const char* jvp_attn_strerror(int code) {
  switch (code) {
    case JVP_OK: return "success";
    case JVP_ERR_INVALID_ARG: return "invalid argument";
    case JVP_ERR_SHAPE_MISMATCH: return "sequence length does not match the mask descriptor";
    case JVP_ERR_UNSUPPORTED_HEAD_DIM: return "unsupported head dimension";
    case JVP_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned";
    case JVP_ERR_LAUNCH_FAILED: return "CUDA launch or runtime error";
    case JVP_ERR_DEVICE_TIMEOUT: return "kernel gave up on a bounded wait";
    case JVP_ERR_DEVICE_BOUNDS: return "kernel saw an out-of-range tile index";
    case JVP_ERR_OUT_OF_MEMORY: return "workspace allocation failed";
    case JVP_ERR_UNSUPPORTED_DEVICE: return "current device is not sm_100";
    case JVP_ERR_TOO_LARGE: return "sizes exceed the kernel's index range";
    default: return "unknown error code";
  }
}

int jvp_attn_version(void) { return JVP_ATTN_VERSION; }

}  // extern "C"
