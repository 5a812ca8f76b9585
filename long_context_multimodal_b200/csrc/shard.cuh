// shard.cuh -- the zigzag shard step: index maps, per-rank modality counts
// and the bit-exact row permute between global and rank-local order.
//
// Source: "LongVILA Guide" (aifetchly), section "Multi-Modal Sequence
// Parallelism (MM-SP) Mechanics", Ring-SP paragraph (each rank holds N/P of
// the tokens). Zigzag reading: 2P chunks of C = N/(2P) tokens, rank r owns
// chunk r then chunk 2P-1-r, which gives every rank the same causal work.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace mmsp {

constexpr int kMaxSegments = 4096;

// Segment table passed by value as a kernel parameter (about 20 KB): segment
// start offsets (n+1 entries, start[n] = N) and kinds.
struct SegTable {
  int32_t n;
  int32_t start[kMaxSegments + 1];
  uint8_t kind[kMaxSegments];
};

// Global position of rank-local slot l (l = r*2C + t).
__device__ __forceinline__ int64_t zigzag_global(int64_t l, int64_t C, int P) {
  int64_t r = l / (2 * C);
  int64_t t = l - r * 2 * C;
  return t < C ? r * C + t : (2 * (int64_t)P - 1 - r) * C + (t - C);
}

// Largest s with start[s] <= g (start[] ascending, start[0] = 0).
__device__ __forceinline__ int seg_of(const int32_t* start, int n, int32_t g) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (start[mid] <= g) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(256) shard_maps_kernel(const __grid_constant__ SegTable tab, int32_t N, int32_t P,
                                                         int32_t* __restrict__ l2g, int32_t* __restrict__ g2l,
                                                         uint8_t* __restrict__ modality,
                                                         int32_t* __restrict__ segid) {
  __shared__ int32_t s_start[kMaxSegments + 1];
  const bool need_seg = (modality != nullptr) || (segid != nullptr);
  if (need_seg) {
    for (int i = threadIdx.x; i <= tab.n; i += blockDim.x) s_start[i] = tab.start[i];
    __syncthreads();
  }
  const int64_t C = N / (2 * P);
  for (int64_t l = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; l < N; l += (int64_t)gridDim.x * blockDim.x) {
    const int32_t g = (int32_t)zigzag_global(l, C, P);
    if (l2g) l2g[l] = g;
    if (g2l) g2l[g] = (int32_t)l;
    if (need_seg) {
      const int s = seg_of(s_start, tab.n, g);
      if (segid) segid[l] = s;
      if (modality) modality[l] = tab.kind[s];
    }
  }
}

// doc_start[g] = first position of the document holding global position g
// (the document table is the segment table of the packed sequence).
__global__ void __launch_bounds__(256) doc_starts_kernel(const __grid_constant__ SegTable tab, int32_t N,
                                                         int32_t* __restrict__ doc_start) {
  __shared__ int32_t s_start[kMaxSegments + 1];
  for (int i = threadIdx.x; i <= tab.n; i += blockDim.x) s_start[i] = tab.start[i];
  __syncthreads();
  for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < N; g += (int64_t)gridDim.x * blockDim.x)
    doc_start[g] = s_start[seg_of(s_start, tab.n, (int32_t)g)];
}

// One block: visual-token prefix over segments, then per rank the text and
// visual counts of its two chunks.
__global__ void __launch_bounds__(256) shard_counts_kernel(const __grid_constant__ SegTable tab, int32_t N,
                                                           int32_t P, int32_t* __restrict__ counts) {
  __shared__ int32_t s_start[kMaxSegments + 1];
  __shared__ int32_t s_vis[kMaxSegments + 1];  // visual tokens before segment s
  for (int i = threadIdx.x; i <= tab.n; i += blockDim.x) s_start[i] = tab.start[i];
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t acc = 0;
    for (int s = 0; s < tab.n; ++s) {
      s_vis[s] = acc;
      if (tab.kind[s]) acc += s_start[s + 1] - s_start[s];
    }
    s_vis[tab.n] = acc;
  }
  __syncthreads();
  const int32_t C = N / (2 * P);
  // visual tokens in [0, g)
  auto vis_before = [&](int32_t g) -> int32_t {
    if (g >= N) return s_vis[tab.n];
    const int s = seg_of(s_start, tab.n, g);
    return s_vis[s] + (tab.kind[s] ? g - s_start[s] : 0);
  };
  for (int r = threadIdx.x; r < P; r += blockDim.x) {
    const int32_t a0 = r * C, b0 = (2 * P - 1 - r) * C;
    const int32_t vis = (vis_before(a0 + C) - vis_before(a0)) + (vis_before(b0 + C) - vis_before(b0));
    counts[2 * r + 0] = 2 * C - vis;
    counts[2 * r + 1] = vis;
  }
}

// Row permute: dst[l] = src[zigzag(l)] (forward) or dst[zigzag(l)] = src[l]
// (inverse). One warp per row, 16-byte vectors; read-only loads.
__global__ void __launch_bounds__(256) shard_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                         int32_t N, int32_t P, int64_t row_vec, int inverse) {
  const int64_t C = N / (2 * P);
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t l = warp; l < N; l += nwarps) {
    const int64_t g = zigzag_global(l, C, P);
    const int64_t sr = inverse ? l : g;
    const int64_t dr = inverse ? g : l;
    const uint4* s = src + sr * row_vec;
    uint4* d = dst + dr * row_vec;
    int64_t i = lane;
    for (; i + 96 < row_vec; i += 128) {
      uint4 a = __ldg(s + i), b = __ldg(s + i + 32), c = __ldg(s + i + 64), e = __ldg(s + i + 96);
      d[i] = a;
      d[i + 32] = b;
      d[i + 64] = c;
      d[i + 96] = e;
    }
    for (; i < row_vec; i += 32) d[i] = __ldg(s + i);
  }
}

// Same permute for rows whose length is a multiple of 4 bytes only.
__global__ void __launch_bounds__(256) shard_rows_words_kernel(const uint32_t* __restrict__ src,
                                                               uint32_t* __restrict__ dst, int32_t N, int32_t P,
                                                               int64_t row_words, int inverse) {
  const int64_t C = N / (2 * P);
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t l = warp; l < N; l += nwarps) {
    const int64_t g = zigzag_global(l, C, P);
    const uint32_t* s = src + (inverse ? l : g) * row_words;
    uint32_t* d = dst + (inverse ? g : l) * row_words;
    for (int64_t i = lane; i < row_words; i += 32) d[i] = __ldg(s + i);
  }
}

}  // namespace mmsp
