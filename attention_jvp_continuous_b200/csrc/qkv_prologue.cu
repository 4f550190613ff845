// Primal-tangent prologue of an attention layer (layer-level JVP, Causal-rCM
// report, Sec. 3.2.2 "JVP FSDP2"): from the fused projections [q | k | v] of
// a token and of its tangent (each H*d channels, head-major), applies RMS
// normalisation to q and k together with its derivative along the tangent,
// rotates both by the token's rotary-embedding row (linear, so the tangent
// rotates like the primal), and writes q, k, v, dq, dk, dv in the [B, H, L,
// d] layout of the attention JVP:
//
//   r  = 1 / sqrt(mean_group(a^2) + eps)
//   y  = a r w,   dy = w r (da - a mean_group(a da) r^2)
//
// Memory-bound: one warp per token; lane l handles the 16-byte vectors
// l + 32 j (8 bf16 channels each) of every block, so a warp reads 512
// contiguous bytes per step and never splits a head's vector. A norm group
// of all H*d channels takes two passes over the token's row (sums, then
// outputs; the second pass hits L1 or L2, and keeping the row in registers
// instead cost occupancy and measured slower); a per-head group (d
// channels) is reduced within the d/8 lanes that hold the head.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace jvp {
namespace prologue {

struct Params {
  const uint4* qkv;   // [B, L, 3 C] bf16 as 16-byte vectors
  const uint4* dqkv;
  uint4* out[6];      // q, k, v, dq, dk, dv: [B, H, L, d]
  const float* norm_w[2];  // q, k weights [group] (null: no norm)
  const float *cos, *sin;  // [L, d/2] (null: no rotation)
  int B, L, H, d, group;
  float eps;
};

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 t = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&t);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Rotates the 4 pairs of a vector by table row `row`, pairs p0 .. p0 + 3.
__device__ __forceinline__ void rotate8(float (&f)[8], const Params& p, int row, int p0) {
  const size_t t = size_t(row) * (p.d / 2) + p0;
  const float4 c = *reinterpret_cast<const float4*>(p.cos + t);
  const float4 s = *reinterpret_cast<const float4*>(p.sin + t);
  const float cc[4] = {c.x, c.y, c.z, c.w}, ss[4] = {s.x, s.y, s.z, s.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float x0 = f[2 * i], x1 = f[2 * i + 1];
    f[2 * i] = fmaf(x0, cc[i], -x1 * ss[i]);
    f[2 * i + 1] = fmaf(x0, ss[i], x1 * cc[i]);
  }
}

// Normalises (optionally), rotates (optionally) and stores one vector of
// block `blk` (0: q, 1: k, 2: v) for token (b, l).
__device__ __forceinline__ void emit(const Params& p, int blk, int b, int l, int vec, float (&x)[8],
                                     float (&dx)[8], bool norm, float r, float dotm, float ms) {
  const int c0 = vec * 8;  // channel within the block
  const int h = c0 / p.d, j0 = c0 % p.d;
  if (norm) {
    const float* w = p.norm_w[blk] + (p.group == p.d ? j0 : c0);
    const float4 w0 = *reinterpret_cast<const float4*>(w);
    const float4 w1 = *reinterpret_cast<const float4*>(w + 4);
    const float ww[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    const float k = dotm / ms;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float y = x[i] * r * ww[i];
      dx[i] = ww[i] * r * fmaf(-x[i], k, dx[i]);
      x[i] = y;
    }
  }
  if (blk < 2 && p.cos) {
    rotate8(x, p, l, j0 / 2);
    rotate8(dx, p, l, j0 / 2);
  }
  const size_t o = ((size_t(b) * p.H + h) * p.L + l) * (p.d / 8) + j0 / 8;
  p.out[blk][o] = pack8(x);
  p.out[3 + blk][o] = pack8(dx);
}

__global__ void __launch_bounds__(256) qkv_prologue_kernel(const Params p) {
  const int lane = threadIdx.x & 31;
  const int C = p.H * p.d;
  const int nvec = C / 8;        // vectors per block of a token
  const int nj = nvec / 32;      // vectors per lane
  const int head_lanes = p.d / 8;  // lanes holding one head (per-head groups)
  const long long n_tok = (long long)p.B * p.L;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long tok = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       tok < n_tok; tok += warps) {
    const int b = int(tok / p.L), l = int(tok % p.L);
    const uint4* row = p.qkv + size_t(tok) * 3 * nvec;
    const uint4* drow = p.dqkv + size_t(tok) * 3 * nvec;
#pragma unroll
    for (int blk = 0; blk < 3; ++blk) {  // unrolled: the pointer arrays take constant indices
      const bool norm = blk < 2 && p.norm_w[blk] != nullptr;
      float r = 1.f, dotm = 0.f, ms = 1.f;
      if (norm && p.group == C) {
        // pass 1: sums over the whole block
        float s2 = 0.f, sd = 0.f;
#pragma unroll 1
        for (int jj = 0; jj < nj; ++jj) {
          float x[8], dx[8];
          unpack8(row[blk * nvec + lane + 32 * jj], x);
          unpack8(drow[blk * nvec + lane + 32 * jj], dx);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            s2 = fmaf(x[i], x[i], s2);
            sd = fmaf(x[i], dx[i], sd);
          }
        }
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) {
          s2 += __shfl_xor_sync(0xffffffffu, s2, m);
          sd += __shfl_xor_sync(0xffffffffu, sd, m);
        }
        ms = s2 / float(C) + p.eps;
        r = 1.f / sqrtf(ms);
        dotm = sd / float(C);
      }
#pragma unroll 1
      for (int jj = 0; jj < nj; ++jj) {
        const int vec = lane + 32 * jj;
        float x[8], dx[8];
        unpack8(row[blk * nvec + vec], x);
        unpack8(drow[blk * nvec + vec], dx);
        if (norm && p.group != C) {
          // per-head group: the head's vectors sit in head_lanes lanes
          float s2 = 0.f, sd = 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            s2 = fmaf(x[i], x[i], s2);
            sd = fmaf(x[i], dx[i], sd);
          }
          for (int m = head_lanes >> 1; m > 0; m >>= 1) {
            s2 += __shfl_xor_sync(0xffffffffu, s2, m);
            sd += __shfl_xor_sync(0xffffffffu, sd, m);
          }
          ms = s2 / float(p.d) + p.eps;
          r = 1.f / sqrtf(ms);
          dotm = sd / float(p.d);
        }
        emit(p, blk, b, l, vec, x, dx, norm, r, dotm, ms);
      }
    }
  }
}

}  // namespace prologue

int launch_qkv_prologue(const PrologueArgs& a, int num_sms) {
  using namespace prologue;
  Params p;
  p.qkv = static_cast<const uint4*>(a.qkv);
  p.dqkv = static_cast<const uint4*>(a.dqkv);
  for (int i = 0; i < 6; ++i) p.out[i] = static_cast<uint4*>(a.out[i]);
  p.norm_w[0] = a.norm_q;
  p.norm_w[1] = a.norm_k;
  p.cos = a.cos;
  p.sin = a.sin;
  p.B = a.B;
  p.L = a.L;
  p.H = a.H;
  p.d = a.d;
  p.group = a.group;
  p.eps = a.eps;
  const long long n_tok = (long long)a.B * a.L;
  const long long blocks = (n_tok + 7) / 8;  // 8 warps (tokens) per block
  const int grid = int(blocks < 8LL * num_sms ? blocks : 8LL * num_sms);
  qkv_prologue_kernel<<<grid, 256, 0, a.stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? JVP_OK : JVP_ERR_LAUNCH_FAILED;
}

}  // namespace jvp
