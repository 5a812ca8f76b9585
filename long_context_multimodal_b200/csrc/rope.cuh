// rope.cuh -- the shard gather of Q / K rows with the rotary position
// embedding applied on the way, and its transpose for the gradients.
//
// Source: "LongVILA Guide" (aifetchly), three-stage curriculum, Stage 2
// (RoPE base raised from 10,000 to 10^7 for long contexts) and section
// "Distributed Training Configuration" (RoPE base 10,000,000). Formula: the
// standard rotary embedding, pair (a, b) of a head vector turned by
// phi_i = pos * theta^(-2i/d): a' = a cos - b sin, b' = a sin + b cos.
// Readings: pairs (i, i + d/2) ("half") or (2i, 2i + 1) ("interleaved");
// pos = global position, or position within the packed document.
//
// One warp per rank-local row; lane k of a head's lane group owns pairs
// 4k..4k+3 and computes their cos / sin once per token for every head of the
// row. The angle is formed and reduced to [-pi, pi] in fp64 (a position of a
// million times a frequency near 1 would lose ~0.05 rad in fp32), then the
// fp32 sine / cosine intrinsics (absolute error ~2^-21 on [-pi, pi]) give
// values far below the bf16 rounding of the result. Rows are rounded to bf16
// with round-to-nearest-even.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "shard.cuh"

namespace mmsp {

constexpr int kRopeMaxPairs = 128;  // d <= 256

struct RopeParams {
  double inv_freq[kRopeMaxPairs];  // theta^(-2i/d), computed on the host in fp64
  int32_t N, P, H;
  int32_t inverse;                 // 0: gather global -> local, +phi; 1: scatter local -> global, -phi
  const int32_t* doc_start;        // [N] global order, or null
};

// Rotate (a, b) by (c, s) and round both to bf16.
__device__ __forceinline__ void rope_rotate(float a, float b, float c, float s, __nv_bfloat16& ra,
                                            __nv_bfloat16& rb) {
  ra = __float2bfloat16_rn(fmaf(a, c, -b * s));
  rb = __float2bfloat16_rn(fmaf(a, s, b * c));
}

template <int D, bool INTERLEAVED>
__global__ void __launch_bounds__(256) shard_rope_kernel(const __grid_constant__ RopeParams p,
                                                         const __nv_bfloat16* __restrict__ src,
                                                         __nv_bfloat16* __restrict__ dst) {
  constexpr int LPH = D / 8;     // lanes per head (each lane: 8 elements = 4 pairs)
  constexpr int HPW = 32 / LPH;  // heads per warp pass
  const int lane = threadIdx.x & 31;
  const int sub = lane % LPH;
  const int hoff = lane / LPH;
  const int64_t C = (int64_t)p.N / (2 * p.P);
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  constexpr double kTwoPi = 6.283185307179586;
  constexpr double kInvTwoPi = 0.15915494309189535;
  for (int64_t l = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); l < p.N; l += warps) {
    const int64_t g = zigzag_global(l, C, p.P);
    const int64_t pos = p.doc_start ? g - (int64_t)p.doc_start[g] : g;
    float cs[4], sn[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const double phi = (double)pos * p.inv_freq[4 * sub + k];
      const double r = fma(-rint(phi * kInvTwoPi), kTwoPi, phi);  // in [-pi, pi] up to rounding
      float sv, cv;
      __sincosf((float)r, &sv, &cv);
      cs[k] = cv;
      sn[k] = p.inverse ? -sv : sv;
    }
    const int64_t srow = p.inverse ? l : g;
    const int64_t drow = p.inverse ? g : l;
    const __nv_bfloat16* sp = src + srow * p.H * D;
    __nv_bfloat16* dp = dst + drow * p.H * D;
    for (int h = hoff; h < p.H; h += HPW) {
      if (INTERLEAVED) {
        // elements 8 sub .. 8 sub + 7 = pairs 4 sub + k as (2k, 2k + 1)
        const uint4 v = *reinterpret_cast<const uint4*>(sp + h * D + 8 * sub);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const __nv_bfloat162 ab = *reinterpret_cast<const __nv_bfloat162*>(&w[k]);
          __nv_bfloat162 r;
          rope_rotate(__low2float(ab), __high2float(ab), cs[k], sn[k], r.x, r.y);
          o[k] = *reinterpret_cast<uint32_t*>(&r);
        }
        *reinterpret_cast<uint4*>(dp + h * D + 8 * sub) = make_uint4(o[0], o[1], o[2], o[3]);
      } else {
        // elements 4 sub .. 4 sub + 3 (first of each pair) and the same + D/2
        const uint2 va = *reinterpret_cast<const uint2*>(sp + h * D + 4 * sub);
        const uint2 vb = *reinterpret_cast<const uint2*>(sp + h * D + D / 2 + 4 * sub);
        const __nv_bfloat162 a01 = *reinterpret_cast<const __nv_bfloat162*>(&va.x);
        const __nv_bfloat162 a23 = *reinterpret_cast<const __nv_bfloat162*>(&va.y);
        const __nv_bfloat162 b01 = *reinterpret_cast<const __nv_bfloat162*>(&vb.x);
        const __nv_bfloat162 b23 = *reinterpret_cast<const __nv_bfloat162*>(&vb.y);
        __nv_bfloat162 ra01, ra23, rb01, rb23;
        rope_rotate(__low2float(a01), __low2float(b01), cs[0], sn[0], ra01.x, rb01.x);
        rope_rotate(__high2float(a01), __high2float(b01), cs[1], sn[1], ra01.y, rb01.y);
        rope_rotate(__low2float(a23), __low2float(b23), cs[2], sn[2], ra23.x, rb23.x);
        rope_rotate(__high2float(a23), __high2float(b23), cs[3], sn[3], ra23.y, rb23.y);
        uint2 oa, ob;
        oa.x = *reinterpret_cast<uint32_t*>(&ra01);
        oa.y = *reinterpret_cast<uint32_t*>(&ra23);
        ob.x = *reinterpret_cast<uint32_t*>(&rb01);
        ob.y = *reinterpret_cast<uint32_t*>(&rb23);
        *reinterpret_cast<uint2*>(dp + h * D + 4 * sub) = oa;
        *reinterpret_cast<uint2*>(dp + h * D + D / 2 + 4 * sub) = ob;
      }
    }
  }
}

}  // namespace mmsp
