// merge.cuh -- the log-sum-exp merge of two partial attention results over
// disjoint key sets (the combine of the ring steps).
//
// The page's ring loop ("LongVILA Guide", section "Implementation",
// LongVILAMultiModalAttention.forward) adds separately normalised blocks;
// the merge used here is the reading that makes the ring equal attention
// over the union of the keys:
//   m = max(la, lb); L = m + ln(e^(la-m) + e^(lb-m)); O = e^(la-L) Oa + e^(lb-L) Ob
// and e^(la-L) = e^(la-m) / (e^(la-m) + e^(lb-m)). Both empty -> (0, -inf).
//
// Layout: o [rows][H][d] fp32, lse [rows][H] fp32. A warp owns 32
// consecutive (row, head) pairs: lane i loads both LSEs of pair i (one
// coalesced 128-byte line per input), computes the weights, and the warp
// then streams the 32 output vectors with 16-byte loads/stores, the weights
// broadcast by warp shuffles.
#pragma once

#include <cstdint>
#include <math_constants.h>

namespace mmsp {

template <int D>
__global__ void __launch_bounds__(256) lse_merge_kernel(const float* o_a, const float* lse_a,
                                                        const float* o_b, const float* lse_b,
                                                        float* o_out, float* lse_out, int64_t total) {
  constexpr int VEC = D / 4;                    // float4 per (row, head)
  constexpr int PER_ITER = 32 / VEC;            // (row, head) pairs per warp step
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const float4* A = reinterpret_cast<const float4*>(o_a);
  const float4* B = reinterpret_cast<const float4*>(o_b);
  float4* O = reinterpret_cast<float4*>(o_out);
  for (int64_t base = warp * 32; base < total; base += nwarps * 32) {
    const int64_t idx = base + lane;
    float wa = 0.f, wb = 0.f;
    if (idx < total) {
      const float la = lse_a[idx], lb = lse_b[idx];
      const float m = fmaxf(la, lb);
      float L = -CUDART_INF_F;
      if (m != -CUDART_INF_F) {
        const float ea = expf(la - m), eb = expf(lb - m);
        const float s = ea + eb;
        L = m + logf(s);
        wa = ea / s;
        wb = eb / s;
      }
      lse_out[idx] = L;
    }
    const int sub = lane / VEC;   // which pair of this step
    const int e = lane % VEC;     // which float4 of the pair
#pragma unroll 4
    for (int j = 0; j < 32; j += PER_ITER) {
      const int jj = j + sub;
      const float wja = __shfl_sync(0xffffffffu, wa, jj);
      const float wjb = __shfl_sync(0xffffffffu, wb, jj);
      const int64_t p = base + jj;
      if (p < total) {
        const float4 x = A[p * VEC + e];
        const float4 y = B[p * VEC + e];
        float4 r;
        r.x = wja * x.x + wjb * y.x;
        r.y = wja * x.y + wjb * y.y;
        r.z = wja * x.z + wjb * y.z;
        r.w = wja * x.w + wjb * y.w;
        O[p * VEC + e] = r;
      }
    }
  }
}

}  // namespace mmsp
