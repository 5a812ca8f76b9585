// ulysses.cuh -- the local data movement around the Ulysses all-to-all of
// 2-D MM-SP: the sequence <-> head transpose.
//
// Source: "LongVILA Guide" (aifetchly), section "Multi-Modal Sequence
// Parallelism (MM-SP) Mechanics" (DeepSpeed Ulysses: (B, N/P, H, D) sequence
// sharded -> (B, N, H/P, D) head sharded by one all_to_all, and back; MM-SP
// factors P = P_u x P_r with Ulysses inside the NVLink domain) and section
// "Implementation", UlyssesAllToAll: the input is split into P_u contiguous
// head groups, group j goes to Ulysses rank j, and the pieces received from
// the P_u ranks are concatenated along the sequence in rank order; the
// inverse splits the sequence and concatenates along the heads.
//
// With rows of `row_bytes` (one head vector) and Hl = H / P_u heads per
// group, on one GPU:
//   pack   (before the forward all-to-all):  dst[j][s][h'] = src[s][j*Hl + h']
//   unpack (after the inverse all-to-all):   dst[s][j*Hl + h'] = src[j][s][h']
// A collective that sends block j of the packed buffer to rank j and lands
// the block from rank i at block i leaves [P_u][S][Hl] = [P_u*S][Hl], the
// head-sharded layout, with no further copy; the inverse sends blocks of the
// head-sharded buffer as they are and unpacks what arrives. pack and unpack
// are inverse permutations, so the backward of either is the other.
//
// Each (s, j) pair moves one contiguous run of Hl * row_bytes bytes: one
// warp per run, 16-byte vector loads and stores (non-coherent loads, the
// source is read once).
#pragma once

#include <cstdint>

namespace mmsp {

__global__ void __launch_bounds__(256) ulysses_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                      int64_t S, int32_t P_u, int64_t run16, int32_t unpack) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t runs = S * P_u;
  for (int64_t w = warp; w < runs; w += nwarps) {
    const int64_t s = w / P_u;
    const int64_t j = w - s * P_u;
    const int64_t seq_major = (s * P_u + j) * run16;   // run (s, j) in [S][H] order
    const int64_t grp_major = (j * S + s) * run16;     // run (j, s) in [P_u][S][Hl] order
    const uint4* a = src + (unpack ? grp_major : seq_major);
    uint4* b = dst + (unpack ? seq_major : grp_major);
    for (int64_t i = lane; i < run16; i += 32) b[i] = __ldg(a + i);
  }
}

}  // namespace mmsp
