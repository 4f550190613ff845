// Row copy with optional rotary position embedding, for key/value caches
// (Causal-rCM report, Sec. 3.2.1 "KV Cache": append mode commits a chunk's
// keys and values into the cache; keys are cached after RoPE, or before it
// and rotated when a read-only forward needs them).
//
// Copies rows [src_row0, src_row0 + rows) of every (b, h) slice of src
// [B, H, src_rows, d] to rows [dst_row0, ...) of dst [B, H, dst_rows, d].
// With tables, row j of the range is rotated by table row rope_row0 + j:
// pairs (x_2i, x_2i+1) -> (x_2i c - x_2i+1 s, x_2i s + x_2i+1 c), c and s
// from cos / sin [rope_rows, d/2] (float32), computed in fp32 and rounded
// once to the element type.
//
// Memory-bound: each thread moves one 16-byte vector per step (8 bf16 or
// 4 fp32 elements, i.e. 4 or 2 pairs) and reads the matching table entries
// (shared by all heads, so they stay in L2); grid-stride over all vectors
// with a grid of a few CTAs per SM.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace jvp {
namespace rope {

template <bool kBf16, bool kRope>
__global__ void __launch_bounds__(256)
rope_copy_kernel(const uint4* src, uint4* dst,  // may be the same rows (in place)
                 const float* __restrict__ cos_t, const float* __restrict__ sin_t, int BH,
                 int src_rows, int dst_rows, int rows, int src_row0, int dst_row0, int vpr,
                 int half_d, int rope_row0) {
  constexpr int kPairs = kBf16 ? 4 : 2;  // pairs per 16-byte vector
  const long long n = (long long)BH * rows * vpr;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < n;
       idx += (long long)gridDim.x * blockDim.x) {
    const int v = int(idx % vpr);
    const long long rr = idx / vpr;
    const int row = int(rr % rows);
    const long long bh = rr / rows;
    uint4 x = src[(bh * src_rows + src_row0 + row) * vpr + v];
    if constexpr (kRope) {
      const size_t t = size_t(rope_row0 + row) * half_d + size_t(v) * kPairs;
      float c[kPairs], s[kPairs];
      if constexpr (kBf16) {
        const float4 c4 = *reinterpret_cast<const float4*>(cos_t + t);
        const float4 s4 = *reinterpret_cast<const float4*>(sin_t + t);
        c[0] = c4.x; c[1] = c4.y; c[2] = c4.z; c[3] = c4.w;
        s[0] = s4.x; s[1] = s4.y; s[2] = s4.z; s[3] = s4.w;
      } else {
        const float2 c2 = *reinterpret_cast<const float2*>(cos_t + t);
        const float2 s2 = *reinterpret_cast<const float2*>(sin_t + t);
        c[0] = c2.x; c[1] = c2.y;
        s[0] = s2.x; s[1] = s2.y;
      }
      uint32_t w[4] = {x.x, x.y, x.z, x.w};
      if constexpr (kBf16) {
#pragma unroll
        for (int k = 0; k < kPairs; ++k) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[k]));
          const float y0 = fmaf(f.x, c[k], -f.y * s[k]);
          const float y1 = fmaf(f.x, s[k], f.y * c[k]);
          const __nv_bfloat162 y = __floats2bfloat162_rn(y0, y1);
          w[k] = *reinterpret_cast<const uint32_t*>(&y);
        }
      } else {
#pragma unroll
        for (int k = 0; k < kPairs; ++k) {
          const float f0 = __uint_as_float(w[2 * k]), f1 = __uint_as_float(w[2 * k + 1]);
          w[2 * k] = __float_as_uint(fmaf(f0, c[k], -f1 * s[k]));
          w[2 * k + 1] = __float_as_uint(fmaf(f0, s[k], f1 * c[k]));
        }
      }
      x = make_uint4(w[0], w[1], w[2], w[3]);
    }
    dst[(bh * dst_rows + dst_row0 + row) * vpr + v] = x;
  }
}

}  // namespace rope

int launch_rope_copy(const RopeArgs& a, int num_sms) {
  using namespace rope;
  if (a.rows == 0) return JVP_OK;
  const bool bf16 = a.bf16;
  const int vpr = a.d / (bf16 ? 8 : 4);
  const long long n = (long long)a.B * a.H * a.rows * vpr;
  const long long blocks = (n + 255) / 256;
  const int grid = int(blocks < 4LL * num_sms ? blocks : 4LL * num_sms);
  const uint4* src = static_cast<const uint4*>(a.src);
  uint4* dst = static_cast<uint4*>(a.dst);
  const int BH = a.B * a.H;
  const bool rot = a.cos != nullptr;
#define JVP_ROPE_LAUNCH(B16, R)                                                           \
  rope_copy_kernel<B16, R><<<grid, 256, 0, a.stream>>>(src, dst, a.cos, a.sin, BH,        \
                                                       a.src_rows, a.dst_rows, a.rows,    \
                                                       a.src_row0, a.dst_row0, vpr,       \
                                                       a.d / 2, a.rope_row0)
  if (bf16 && rot) JVP_ROPE_LAUNCH(true, true);
  else if (bf16) JVP_ROPE_LAUNCH(true, false);
  else if (rot) JVP_ROPE_LAUNCH(false, true);
  else JVP_ROPE_LAUNCH(false, false);
#undef JVP_ROPE_LAUNCH
  return cudaGetLastError() == cudaSuccess ? JVP_OK : JVP_ERR_LAUNCH_FAILED;
}

}  // namespace jvp
