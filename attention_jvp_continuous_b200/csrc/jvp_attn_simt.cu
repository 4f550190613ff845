// CUDA-core masked attention JVP (fp32 arithmetic).
//
// One warp per query row. Keys are streamed in groups of 32 through the
// row's admissible intervals only (Causal-rCM report, Appendix B: the same
// range list drives the score and its tangent). Each group updates the
// online-softmax state {m, l, g = sum e*dS} and the accumulators
// A1 = sum e V and A23 = sum e dS V + sum e dV, all rescaled by the same
// factor exp(m_old - m_new) (Appendix B, text after Eq. 45). The finish is
//   O = A1 / l,  mu = g / l,  dO = A23 / l - mu O,  LSE = m + log l.
// Lane t owns output columns t, t+32, t+64, t+96.
//
// This path serves fp32 inputs (where bf16 tensor-core operands could not
// meet a 1e-4 relative tolerance) and head dims other than 128.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "common.cuh"
#include "mask_rows.cuh"

namespace jvp {
namespace {

constexpr int kRowsPerBlock = 8;  // one warp per row

__device__ __forceinline__ float load_f(const float* p) { return *p; }
__device__ __forceinline__ float load_f(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
__device__ __forceinline__ void store_f(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_f(__nv_bfloat16* p, float x) {
  *p = __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <typename T, int NT>
__global__ void __launch_bounds__(kRowsPerBlock * 32)
jvp_attn_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                     const T* __restrict__ v, const T* __restrict__ dq,
                     const T* __restrict__ dk, const T* __restrict__ dv,
                     T* __restrict__ o, T* __restrict__ d_o,
                     float* __restrict__ lse, int L, int row_blocks,
                     jvp_mask_desc mask, float scale) {
  constexpr int D = NT * 32;
  __shared__ float sq[kRowsPerBlock][D];
  __shared__ float sdq[kRowsPerBlock][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x / row_blocks;
  const int row = (blockIdx.x % row_blocks) * kRowsPerBlock + warp;
  if (row >= L) return;  // whole warp leaves together; no block barrier below
  const size_t base = size_t(bh) * L * D;
  const size_t qoff = base + size_t(row) * D;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    sq[warp][lane + 32 * t] = load_f(q + qoff + lane + 32 * t);
    sdq[warp][lane + 32 * t] = load_f(dq + qoff + lane + 32 * t);
  }
  __syncwarp();

  const int chunk = mask.chunk < 1 ? 1 : mask.chunk;
  const RowKeys rk = row_keys(mask.mode, mask.tokens_per_frame, mask.n_frames,
                              chunk, L, row);
  float m = -CUDART_INF_F, l = 0.f, g = 0.f;
  float a1[NT], a23[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) a1[t] = a23[t] = 0.f;

  for (int iv = 0; iv < 2; ++iv) {
    const int lo = iv == 0 ? rk.a0 : rk.a1;
    const int hi = iv == 0 ? rk.b0 : rk.b1;
    for (int j0 = lo; j0 < hi; j0 += 32) {
      const int j = j0 + lane;
      const bool ok = j < hi;
      float s = -CUDART_INF_F, ds = 0.f;
      if (ok) {
        const T* kr = k + base + size_t(j) * D;
        const T* dkr = dk + base + size_t(j) * D;
        float acc = 0.f, dacc = 0.f;
#pragma unroll 8
        for (int t = 0; t < D; ++t) {
          const float kv = load_f(kr + t);
          acc = fmaf(sq[warp][t], kv, acc);
          dacc = fmaf(sdq[warp][t], kv, dacc);
          dacc = fmaf(sq[warp][t], load_f(dkr + t), dacc);
        }
        s = acc * scale;
        ds = dacc * scale;
      }
      // j0 < hi, so lane 0 is admitted and the group maximum is finite.
      const float mn = fmaxf(m, warp_max(s));
      const float alpha = (m == -CUDART_INF_F) ? 0.f : expf(m - mn);
      const float e = ok ? expf(s - mn) : 0.f;
      const float eds = e * ds;
      l = l * alpha + warp_sum(e);
      g = g * alpha + warp_sum(eds);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        a1[t] *= alpha;
        a23[t] *= alpha;
      }
      const int cnt = min(32, hi - j0);
      for (int jj = 0; jj < cnt; ++jj) {
        const float ej = __shfl_sync(0xffffffffu, e, jj);
        const float edj = __shfl_sync(0xffffffffu, eds, jj);
        const size_t roff = base + size_t(j0 + jj) * D;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const float vv = load_f(v + roff + lane + 32 * t);
          const float dvv = load_f(dv + roff + lane + 32 * t);
          a1[t] = fmaf(ej, vv, a1[t]);
          a23[t] = fmaf(edj, vv, fmaf(ej, dvv, a23[t]));
        }
      }
      m = mn;
    }
  }

  const float inv = l > 0.f ? 1.f / l : 0.f;
  const float mu = g * inv;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const float ov = a1[t] * inv;
    store_f(o + qoff + lane + 32 * t, ov);
    store_f(d_o + qoff + lane + 32 * t, a23[t] * inv - mu * ov);
  }
  if (lane == 0)
    lse[size_t(bh) * L + row] = l > 0.f ? m + logf(l) : -CUDART_INF_F;
}

template <typename T>
int launch_t(const LaunchArgs& a) {
  const int row_blocks = (a.L + kRowsPerBlock - 1) / kRowsPerBlock;
  const long long blocks = (long long)row_blocks * a.B * a.H;
  if (blocks > 0x7fffffffLL) return JVP_ERR_TOO_LARGE;
  dim3 grid((unsigned)blocks), block(kRowsPerBlock * 32);
#define JVP_SIMT_CASE(NT)                                                     \
  case NT:                                                                    \
    jvp_attn_simt_kernel<T, NT><<<grid, block, 0, a.stream>>>(                \
        (const T*)a.q, (const T*)a.k, (const T*)a.v, (const T*)a.dq,          \
        (const T*)a.dk, (const T*)a.dv, (T*)a.o, (T*)a.d_o, a.lse, a.L,       \
        row_blocks, a.mask, a.scale);                                         \
    break;
  switch (a.d / 32) {
    JVP_SIMT_CASE(1)
    JVP_SIMT_CASE(2)
    JVP_SIMT_CASE(3)
    JVP_SIMT_CASE(4)
    default:
      return JVP_ERR_UNSUPPORTED_HEAD_DIM;
  }
#undef JVP_SIMT_CASE
  return cudaGetLastError() == cudaSuccess ? JVP_OK : JVP_ERR_LAUNCH_FAILED;
}

}  // namespace

int launch_simt(const LaunchArgs& a, bool bf16) {
  if (a.d % 32 != 0 || a.d < 32 || a.d > 128) return JVP_ERR_UNSUPPORTED_HEAD_DIM;
  return bf16 ? launch_t<__nv_bfloat16>(a) : launch_t<float>(a);
}

}  // namespace jvp
