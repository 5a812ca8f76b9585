// ring.cuh -- ring-order bookkeeping shared by the attention kernels.
//
// In ring attention ("LongVILA Guide" (aifetchly), section "Implementation",
// LongVILAMultiModalAttention.forward and LongVILAParallelContext) rank r
// holds, at ring step s, the K/V block that rank (r - s) mod P started
// with; with zigzag sharding every rank's block is two chunks (chunk k and
// chunk 2P-1-k of the sequence for rank k). The kernels walk the steps in
// order and, within a step, the rank's two chunks in order.
#pragma once

#include <cstdint>

namespace mmsp {

// Up to four ring visits (step s, chunk ck of the rank held at step s),
// ascending in (s, ck) -- the ring order -- packed as 16-bit codes 2s + ck
// (0xFFFF: none). Used by packed-document iterators, whose items see only
// the few chunks that hold their documents, instead of walking every step.
struct RingList {
  uint64_t codes;
  int n;  // entries left; -1: not used (walk every step)

  // Chunks [c0, c1] (global chunk indices, c1 - c0 < 4) seen from a rank
  // whose partner at step s is rank (base + sign * s) mod P.
  __device__ __forceinline__ void build(int c0, int c1, int P, int base, int sign, int s_begin, int s_end) {
    n = -1;
    codes = ~0ull;
    if (c1 - c0 >= 4 || 2 * P >= 0xFFFF) return;
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int g = c0 + i;
      c[i] = 0xFFFFu;
      if (g <= c1) {
        const int k = g < P ? g : 2 * P - 1 - g;    // rank that owns chunk g
        int st = sign > 0 ? (k - base) % P : (base - k) % P;
        if (st < 0) st += P;
        if (st >= s_begin && st < s_end) c[i] = (uint32_t)(2 * st + (g < P ? 0 : 1));
      }
    }
    // sorting network on four values
    auto cs = [](uint32_t& a, uint32_t& b) {
      const uint32_t lo = a < b ? a : b, hi = a < b ? b : a;
      a = lo;
      b = hi;
    };
    cs(c[0], c[1]);
    cs(c[2], c[3]);
    cs(c[0], c[2]);
    cs(c[1], c[3]);
    cs(c[1], c[2]);
    n = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) n += c[i] != 0xFFFFu ? 1 : 0;
    codes = (uint64_t)c[0] | ((uint64_t)c[1] << 16) | ((uint64_t)c[2] << 32) | ((uint64_t)c[3] << 48);
  }

  __device__ __forceinline__ bool pop(int& step, int& chunk) {
    if (n <= 0) return false;
    const uint32_t code = (uint32_t)(codes & 0xFFFFu);
    codes >>= 16;
    --n;
    step = (int)(code >> 1);
    chunk = (int)(code & 1u);
    return true;
  }
};

}  // namespace mmsp
