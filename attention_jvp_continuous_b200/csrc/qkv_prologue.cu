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
// contiguous bytes per step and never splits a head's vector. For H*d up to
// 2048 channels (8 vectors per lane) qkv_prologue_reg_kernel holds a block
// in registers; wider layers take qkv_prologue_kernel, where a norm group of
// all H*d channels takes two passes over the token's row (sums, then
// outputs; the second pass hits L1 or L2). A per-head group (d channels)
// is reduced within the d/8 lanes that hold the head.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "sm100_ptx.cuh"

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

// Streaming 16-byte load: each projection vector is read exactly once.
__device__ __forceinline__ uint4 ld_stream(const uint4* ptr) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(ptr));
  return r;
}

// Register-resident form for blocks of NJ = H*d / 256 <= 8 vectors per lane.
// A lane loads all NJ vectors of x and of dx of a block before using any of
// them, so a warp has 2 * NJ * 512 bytes in flight, and the full-width norm
// needs no second pass over the row. Because d is a power of two dividing
// 256, every vector of a lane sits at the same dimension j0 = 8 lane mod d
// of its head: the lane's rotation pairs (one table row per token) and, for
// per-head groups, its norm weights are loaded once and reused for q and k,
// x and dx. v is a pure layout change and is copied without conversion.
template <int NJ>
__global__ void __launch_bounds__(256) qkv_prologue_reg_kernel(const Params p) {
  const int lane = threadIdx.x & 31;
  const int dshift = 31 - __clz(p.d);
  const int C = p.H << dshift;
  const int nvec = C >> 3;
  const int head_lanes = p.d >> 3;
  const int j0 = (lane * 8) & (p.d - 1);
  const bool rope = p.cos != nullptr;
  const bool norm = p.norm_w[0] != nullptr;
  const bool head_norm = norm && p.group != C;
  float wh[2][8];  // per-head norm weights of q and k at dimensions j0 .. j0 + 7
#pragma unroll
  for (int blk = 0; blk < 2; ++blk) {
#pragma unroll
    for (int i = 0; i < 8; ++i) wh[blk][i] = 1.f;
    if (head_norm) {
      const float4 w0 = *reinterpret_cast<const float4*>(p.norm_w[blk] + j0);
      const float4 w1 = *reinterpret_cast<const float4*>(p.norm_w[blk] + j0 + 4);
      wh[blk][0] = w0.x; wh[blk][1] = w0.y; wh[blk][2] = w0.z; wh[blk][3] = w0.w;
      wh[blk][4] = w1.x; wh[blk][5] = w1.y; wh[blk][6] = w1.z; wh[blk][7] = w1.w;
    }
  }
  const long long n_tok = (long long)p.B * p.L;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long tok = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       tok < n_tok; tok += warps) {
    const int b = int(tok / p.L), l = int(tok % p.L);
    const uint4* row = p.qkv + size_t(tok) * 3 * nvec;
    const uint4* drow = p.dqkv + size_t(tok) * 3 * nvec;
    // Output vector index of (head h, this token, dimension j0).
    const size_t obase = (size_t(b) * p.H * p.L + l) * (p.d >> 3) + (j0 >> 3);
    const size_t ohead = size_t(p.L) * (p.d >> 3);
    float cs[4], sn[4];
    if (rope) {
      const size_t t = size_t(l) * (p.d >> 1) + (j0 >> 1);
      const float4 c = *reinterpret_cast<const float4*>(p.cos + t);
      const float4 s = *reinterpret_cast<const float4*>(p.sin + t);
      cs[0] = c.x; cs[1] = c.y; cs[2] = c.z; cs[3] = c.w;
      sn[0] = s.x; sn[1] = s.y; sn[2] = s.z; sn[3] = s.w;
    }
#pragma unroll
    for (int blk = 0; blk < 2; ++blk) {  // q, k
      uint4 xv[NJ], dv[NJ];
#pragma unroll
      for (int jj = 0; jj < NJ; ++jj) {
        xv[jj] = ld_stream(row + blk * nvec + lane + 32 * jj);
        dv[jj] = ld_stream(drow + blk * nvec + lane + 32 * jj);
      }
      float r = 1.f, k = 0.f;
      if (norm && !head_norm) {
        float s2 = 0.f, sd = 0.f;
#pragma unroll
        for (int jj = 0; jj < NJ; ++jj) {
          float x[8], dx[8];
          unpack8(xv[jj], x);
          unpack8(dv[jj], dx);
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
        const float ms = s2 / float(C) + p.eps;
        r = 1.f / sqrtf(ms);
        k = (sd / float(C)) / ms;
      }
#pragma unroll
      for (int jj = 0; jj < NJ; ++jj) {
        const int vec = lane + 32 * jj;
        float x[8], dx[8];
        unpack8(xv[jj], x);
        unpack8(dv[jj], dx);
        if (head_norm) {
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
          const float ms = s2 / float(p.d) + p.eps;
          r = 1.f / sqrtf(ms);
          k = (sd / float(p.d)) / ms;
        }
        if (norm) {
          // y = a (r w), dy = (r w) (da - a k), k = mean(a da) r^2, in
          // packed pairs.
          float w[8];
          if (head_norm) {
#pragma unroll
            for (int i = 0; i < 8; ++i) w[i] = wh[blk][i];
          } else {
            const float4 w0 = *reinterpret_cast<const float4*>(p.norm_w[blk] + vec * 8);
            const float4 w1 = *reinterpret_cast<const float4*>(p.norm_w[blk] + vec * 8 + 4);
            w[0] = w0.x; w[1] = w0.y; w[2] = w0.z; w[3] = w0.w;
            w[4] = w1.x; w[5] = w1.y; w[6] = w1.z; w[7] = w1.w;
          }
          const uint64_t r2 = ptx::f2pack(r, r), nk2 = ptx::f2pack(-k, -k);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint64_t rw = ptx::mul2(r2, ptx::f2pack(w[2 * i], w[2 * i + 1]));
            const uint64_t xp = ptx::f2pack(x[2 * i], x[2 * i + 1]);
            const uint64_t t = ptx::fma2(xp, nk2, ptx::f2pack(dx[2 * i], dx[2 * i + 1]));
            ptx::f2unpack(ptx::mul2(xp, rw), x[2 * i], x[2 * i + 1]);
            ptx::f2unpack(ptx::mul2(rw, t), dx[2 * i], dx[2 * i + 1]);
          }
        }
        if (rope) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float x0 = x[2 * i], x1 = x[2 * i + 1];
            x[2 * i] = fmaf(x0, cs[i], -x1 * sn[i]);
            x[2 * i + 1] = fmaf(x0, sn[i], x1 * cs[i]);
            const float d0 = dx[2 * i], d1 = dx[2 * i + 1];
            dx[2 * i] = fmaf(d0, cs[i], -d1 * sn[i]);
            dx[2 * i + 1] = fmaf(d0, sn[i], d1 * cs[i]);
          }
        }
        const size_t o = obase + size_t((vec * 8) >> dshift) * ohead;
        p.out[blk][o] = pack8(x);
        p.out[3 + blk][o] = pack8(dx);
      }
    }
    {  // v: layout change only
      uint4 xv[NJ], dv[NJ];
#pragma unroll
      for (int jj = 0; jj < NJ; ++jj) {
        xv[jj] = ld_stream(row + 2 * nvec + lane + 32 * jj);
        dv[jj] = ld_stream(drow + 2 * nvec + lane + 32 * jj);
      }
#pragma unroll
      for (int jj = 0; jj < NJ; ++jj) {
        const size_t o = obase + size_t(((lane + 32 * jj) * 8) >> dshift) * ohead;
        p.out[2][o] = xv[jj];
        p.out[5][o] = dv[jj];
      }
    }
  }
}

// Persistent grid: as many 256-thread blocks as fit on the SMs at once, so
// that every block is resident and takes an equal share of the tokens.
template <class K>
static int launch_resident(K kernel, const Params& p, long long n_tok, int num_sms,
                           cudaStream_t st) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, 256, 0) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const long long blocks = (n_tok + 7) / 8;  // 8 warps (tokens) per block
  const long long cap = (long long)per_sm * num_sms;
  const int grid = int(blocks < cap ? blocks : cap);
  kernel<<<grid, 256, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? JVP_OK : JVP_ERR_LAUNCH_FAILED;
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
  switch (a.H * a.d / 256) {  // vectors of a block per lane
    case 1: return launch_resident(qkv_prologue_reg_kernel<1>, p, n_tok, num_sms, a.stream);
    case 2: return launch_resident(qkv_prologue_reg_kernel<2>, p, n_tok, num_sms, a.stream);
    case 3: return launch_resident(qkv_prologue_reg_kernel<3>, p, n_tok, num_sms, a.stream);
    case 4: return launch_resident(qkv_prologue_reg_kernel<4>, p, n_tok, num_sms, a.stream);
    case 5: return launch_resident(qkv_prologue_reg_kernel<5>, p, n_tok, num_sms, a.stream);
    case 6: return launch_resident(qkv_prologue_reg_kernel<6>, p, n_tok, num_sms, a.stream);
    case 7: return launch_resident(qkv_prologue_reg_kernel<7>, p, n_tok, num_sms, a.stream);
    case 8: return launch_resident(qkv_prologue_reg_kernel<8>, p, n_tok, num_sms, a.stream);
    default: break;
  }
  const long long blocks = (n_tok + 7) / 8;  // 8 warps (tokens) per block
  const int grid = int(blocks < 8LL * num_sms ? blocks : 8LL * num_sms);
  qkv_prologue_kernel<<<grid, 256, 0, a.stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? JVP_OK : JVP_ERR_LAUNCH_FAILED;
}

}  // namespace jvp
