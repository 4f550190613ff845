// jvp_attn_fwd_noalloc: the tensor-core masked attention JVP for callers
// that must not allocate device memory.
//
// jvp_attn_fwd keeps the tile work list of each (mask, L) in a device
// buffer that it allocates with cudaMalloc on first use. Some callers cannot
// allow that: frameworks whose device memory all belongs to their own pool
// or arena, and deployments that forbid device allocation after start-up
// (a cudaMalloc may also synchronise the device). This variant keeps the
// work list in a fixed array in the library's own device memory instead,
// g_noalloc_worklist below, and otherwise runs the same kernel.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds it (256 KiB) until the process exits. Host code may not use
// its name as a device address; the address is looked up once per device
// with cudaGetSymbolAddress while that device is current.
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "common.cuh"
#include "schedule.h"

namespace {

// Size of the scratch array, in int32 words. The first kCounterWords hold
// the kernel's work-item counter (zeroed on the stream before every launch);
// the work list follows: 4 words per 128-row query tile plus 2 per key-tile
// segment. The teacher-forcing mask at 1560 tokens per frame needs about 81
// words per 1000 tokens, so the list fits up to roughly 800,000 tokens.
constexpr int64_t kNoallocWords = 65536;
constexpr int64_t kCounterWords = 64;  // keeps the list 256-byte aligned
constexpr int64_t kListWords = kNoallocWords - kCounterWords;
constexpr int kBM = 128, kBN = 64;
constexpr int kMaxDevices = 64;

// Device scratch shared by every call on a device.
static __device__ __align__(256) int32_t g_noalloc_worklist[kNoallocWords];
// Host staging for the list before it is copied into g_noalloc_worklist.
static int32_t g_noalloc_host[kListWords];

struct NoallocDev {
  bool ready = false;
  int32_t* scratch = nullptr;  // device address of g_noalloc_worklist
  int32_t* list = nullptr;     // scratch + kCounterWords
  bool have = false;           // key of the list the scratch currently holds
  int mode = 0, T = 0, F = 0, chunk = 0, L = 0;
  int n_qt = 0, n_segs = 0;
};

std::mutex g_na_mu;
NoallocDev g_na[kMaxDevices];

}  // namespace

extern "C" int jvp_attn_fwd_noalloc(const void* q, const void* k, const void* v, const void* dq,
                                    const void* dk, const void* dv, void* o, void* d_o,
                                    float* lse, int B, int H, int L, int d, jvp_dtype dtype,
                                    jvp_mask_desc mask, float softmax_scale, void* stream) {
  using namespace jvp;
  if (!q || !k || !v || !dq || !dk || !dv || !o || !d_o || !lse) return JVP_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || L <= 0 || d <= 0 || dtype != JVP_BF16) return JVP_ERR_INVALID_ARG;
  if (std::isnan(softmax_scale) || std::isinf(softmax_scale)) return JVP_ERR_INVALID_ARG;
  if (d != 128) return JVP_ERR_UNSUPPORTED_HEAD_DIM;
  int rc = validate_mask(mask, L);
  if (rc != JVP_OK) return rc;
  if ((long long)B * H * L >= (1LL << 31) || (long long)B * H >= (1LL << 31) / 2)
    return JVP_ERR_TOO_LARGE;
  const void* ptrs[] = {q, k, v, dq, dk, dv, o, d_o, lse};
  for (const void* p : ptrs)
    if (reinterpret_cast<uintptr_t>(p) & 15u) return JVP_ERR_MISALIGNED;
  // Query-tile entries alone must fit before the list is worth building.
  if (4LL * ((L + kBM - 1) / kBM) > kListWords) return JVP_ERR_TOO_LARGE;

  int sms = 0;
  unsigned* err = nullptr;
  rc = current_device_state(&sms, &err);
  if (rc != JVP_OK) return rc;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return JVP_ERR_LAUNCH_FAILED;
  if (dev < 0 || dev >= kMaxDevices) return JVP_ERR_UNSUPPORTED_DEVICE;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The cached (mask, L) key below lives on the host. A call recorded into
  // a graph on a cache hit would bake in the list sizes of that moment and
  // replay against whatever list a later call left in the array, so calls
  // on a capturing stream are refused. A failed query (e.g. the legacy
  // stream while another stream captures globally) is refused too.
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) {
    cudaGetLastError();
    return JVP_ERR_INVALID_ARG;
  }
  if (cap != cudaStreamCaptureStatusNone) return JVP_ERR_INVALID_ARG;
  WorkList w;
  unsigned* counter = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_na_mu);
    NoallocDev& s = g_na[dev];
    if (!s.ready) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_worklist) != cudaSuccess) {
        cudaGetLastError();
        return JVP_ERR_LAUNCH_FAILED;
      }
      s.scratch = static_cast<int32_t*>(p);
      s.list = s.scratch + kCounterWords;
      s.ready = true;
    }
    const bool same = s.have && s.mode == mask.mode && s.T == mask.tokens_per_frame &&
                      s.F == mask.n_frames && s.chunk == mask.chunk && s.L == L;
    if (!same) {
      const int n_qt = (L + kBM - 1) / kBM;
      int nq = 0, ns = 0;
      const int64_t seg_off = 4LL * n_qt;
      if (!build_schedule_into(mask, L, kBM, kBN, g_noalloc_host, seg_off,
                               g_noalloc_host + seg_off, kListWords - seg_off, &nq, &ns))
        return JVP_ERR_TOO_LARGE;
      // The scratch is rewritten in stream order; it no longer holds the
      // previous list even if this call fails later.
      s.have = false;
      const size_t bytes = size_t(seg_off + 2LL * ns) * sizeof(int32_t);
      if (cudaMemcpyAsync(s.list, g_noalloc_host, bytes, cudaMemcpyHostToDevice, st) !=
          cudaSuccess)
        return JVP_ERR_LAUNCH_FAILED;
      s.have = true;
      s.mode = mask.mode;
      s.T = mask.tokens_per_frame;
      s.F = mask.n_frames;
      s.chunk = mask.chunk;
      s.L = L;
      s.n_qt = nq;
      s.n_segs = ns;
    }
    w.qtiles = reinterpret_cast<const int4*>(s.list);
    w.segs = reinterpret_cast<const int2*>(s.list + 4LL * s.n_qt);
    counter = reinterpret_cast<unsigned*>(s.scratch);
    w.n_qtiles = s.n_qt;
    w.n_segs = s.n_segs;
  }

  LaunchArgs a;
  a.q = q; a.k = k; a.v = v; a.dq = dq; a.dk = dk; a.dv = dv;
  a.o = o; a.d_o = d_o; a.lse = lse;
  a.B = B; a.H = H; a.L = L; a.d = d;
  a.mask = mask;
  a.scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(float(d));
  a.stream = st;
  a.err = err;
  a.item_ctr = counter;
  a.wait_limit_ns = wait_limit_ns();
  a.stall_test = stall_test();
  return launch_sm100(a, w, sms);
}
