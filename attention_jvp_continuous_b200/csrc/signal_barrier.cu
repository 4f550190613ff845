// Device-side barrier of the ranks of a context-parallel group, one process
// per GPU, ordered on a stream (the synchronisation around the fused output
// exchange of Ulysses context parallelism, Causal-rCM report, Sec. 3.2.2
// "JVP Ulysses CP": the ranks' kernels store rows into each other's shards,
// so a rank may neither overwrite a shard its owner still reads nor read
// its own shard before every rank's stores have landed).
//
// Every rank owns n flag words that all ranks can reach (symmetric memory
// or peer mappings). At barrier number `epoch` rank r, once the work before
// the barrier on its stream is complete, release-stores epoch into word r
// of every rank's flags, then waits with acquire loads until each of its own
// n words has reached epoch. The wait is bounded: past the library's wait
// limit the kernel records a timeout in the device error word and returns,
// so a rank that never arrives shows up as JVP_ERR_DEVICE_TIMEOUT on the
// host instead of a hang.
#include <cuda_runtime.h>

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace jvp {
namespace barrier {

struct Params {
  uint32_t* flags[kMaxShards];  // flags[q]: rank q's words, as this process addresses them
  int n, rank;
  uint32_t epoch;
  unsigned* err;
  unsigned long long limit_ns;
};

__global__ void __launch_bounds__(32) signal_barrier_kernel(const Params p) {
  const int q = threadIdx.x;
  if (q < p.n) {
    // Release at system scope: the stores of the work that preceded this
    // launch on the stream (other kernels included) are visible to rank q
    // before it sees the flag.
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p.flags[q] + p.rank), "r"(p.epoch)
                 : "memory");
    const uint32_t* mine = p.flags[p.rank] + q;
    const uint64_t t0 = ptx::globaltimer();
    for (uint32_t it = 0;; ++it) {
      uint32_t v;
      asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(mine) : "memory");
      if (int32_t(v - p.epoch) >= 0) break;  // wrap-around safe
      if ((it & 15u) == 15u && ptx::globaltimer() - t0 > p.limit_ns) {
        atomicOr(p.err, kErrTimeout);
        break;
      }
      __nanosleep(64);
    }
  }
}

}  // namespace barrier

int launch_signal_barrier(uint32_t* const* flags, int n, int rank, uint32_t epoch,
                          unsigned* err, unsigned long long limit_ns, cudaStream_t st) {
  barrier::Params p{};
  for (int q = 0; q < n; ++q) p.flags[q] = flags[q];
  p.n = n;
  p.rank = rank;
  p.epoch = epoch;
  p.err = err;
  p.limit_ns = limit_ns;
  barrier::signal_barrier_kernel<<<1, 32, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? JVP_OK : JVP_ERR_LAUNCH_FAILED;
}

}  // namespace jvp
