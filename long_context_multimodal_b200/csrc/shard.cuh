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

// ----------------------------------------------------------------------------
// Frame-aligned, modality-balanced encoder shard ("LongVILA Guide" (aifetchly),
// section "Problem": modality-switching boundaries leave one rank with pure
// text and another with dense visual patches). Reading: frame f (a visual
// segment) goes whole to encoder rank floor(P * V_f / V), V_f = visual tokens
// before it; text token t (text tokens counted alone) to rank floor(P * t /
// T); the encoder layout is rank 0's frames then its text, rank 1's frames
// then its text, and so on. With vis_start(e) = V_f of rank e's first frame
// (V when none) and txt_start(e) = ceil(e * T / P), a visual token with
// visual index v on rank e sits at row txt_start(e) + v, and a text token
// with text index t on rank e at row vis_start(e + 1) + t.

// Visual tokens before each segment (s_vis[0..n], s_vis[n] = V), by a
// block-wide scan over the table: each thread sums a contiguous run of
// segments, thread 0 scans the run totals, each thread writes its run.
__device__ __forceinline__ void visual_prefix(const SegTable& tab, const int32_t* s_start, int32_t* s_vis,
                                              int32_t* s_part) {
  const int n = tab.n;
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int a = threadIdx.x * per, b = min(n, a + per);
  int32_t sum = 0;
  for (int i = a; i < b; ++i) sum += tab.kind[i] ? s_start[i + 1] - s_start[i] : 0;
  s_part[threadIdx.x] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t acc = 0;
    for (int i = 0; i < (int)blockDim.x; ++i) {
      const int32_t x = s_part[i];
      s_part[i] = acc;
      acc += x;
    }
  }
  __syncthreads();
  int32_t acc = s_part[threadIdx.x];
  for (int i = a; i < b; ++i) {
    s_vis[i] = acc;
    acc += tab.kind[i] ? s_start[i + 1] - s_start[i] : 0;
  }
  if (b == n && a < b) s_vis[n] = acc;
  if (n == 0 && threadIdx.x == 0) s_vis[0] = 0;
  __syncthreads();
}

struct FramePlan {
  const int32_t* start;  // shared: segment starts
  const int32_t* vis;    // shared: visual tokens before each segment
  const uint8_t* kind;   // segment kinds
  int n, P;
  int32_t V, T;

  // V_f of the first frame whose rank is >= x (V when there is none).
  __device__ __forceinline__ int32_t vis_start(int x) const {
    const int64_t X = ((int64_t)x * V + P - 1) / P;
    int lo = 0, hi = n;  // first s with vis[s] >= X (vis[n] = V >= X)
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (vis[mid] >= X) hi = mid;
      else lo = mid + 1;
    }
    return vis[lo];
  }
  __device__ __forceinline__ int32_t txt_start(int x) const {
    return (int32_t)(((int64_t)x * T + P - 1) / P);
  }
  __device__ __forceinline__ int32_t row(int32_t g) const {
    const int s = seg_of(start, n, g);
    if (kind[s]) {
      const int e = (int)(((int64_t)P * vis[s]) / V);
      return txt_start(e) + vis[s] + (g - start[s]);
    }
    const int32_t t = g - vis[s];
    const int e = (int)(((int64_t)P * t) / T);
    return vis_start(e + 1) + t;
  }
};

__global__ void __launch_bounds__(256) frame_maps_kernel(const __grid_constant__ SegTable tab, int32_t N, int32_t P,
                                                         int32_t* __restrict__ global2enc,
                                                         int32_t* __restrict__ local2enc,
                                                         int32_t* __restrict__ counts) {
  __shared__ int32_t s_start[kMaxSegments + 1];
  __shared__ int32_t s_vis[kMaxSegments + 1];
  __shared__ int32_t s_part[256];
  for (int i = threadIdx.x; i <= tab.n; i += blockDim.x) s_start[i] = tab.start[i];
  __syncthreads();
  visual_prefix(tab, s_start, s_vis, s_part);
  FramePlan fp{s_start, s_vis, tab.kind, tab.n, P, s_vis[tab.n], N - s_vis[tab.n]};
  const int64_t C = N / (2 * P);
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < N; i += (int64_t)gridDim.x * blockDim.x) {
    if (global2enc) global2enc[i] = fp.row((int32_t)i);
    if (local2enc) local2enc[i] = fp.row((int32_t)zigzag_global(i, C, P));
  }
  if (counts && blockIdx.x == 0) {
    for (int e = threadIdx.x; e < P; e += blockDim.x) {
      counts[2 * e + 0] = fp.vis_start(e + 1) - fp.vis_start(e);
      counts[2 * e + 1] = fp.txt_start(e + 1) - fp.txt_start(e);
    }
  }
}

// Indexed row copy: dst[i] = src[index[i]] (gather) or dst[index[i]] =
// src[i] (scatter), rows of row_vec 16-byte vectors; one warp per row. An
// index outside [0, n_rows) is skipped and recorded (error word 3).
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                          const int32_t* __restrict__ index, int64_t n_rows,
                                                          int64_t row_vec, int scatter) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t i = warp; i < n_rows; i += nwarps) {
    const int64_t j = __ldg(index + i);
    if (j < 0 || j >= n_rows) {
      if (lane == 0) atomicExch(&g_timeout_flag, 3);
      continue;
    }
    const uint4* a = src + (scatter ? i : j) * row_vec;
    uint4* b = dst + (scatter ? j : i) * row_vec;
    for (int64_t k = lane; k < row_vec; k += 32) b[k] = __ldg(a + k);
  }
}

}  // namespace mmsp
