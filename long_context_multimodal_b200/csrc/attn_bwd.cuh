// attn_bwd.cuh -- gradients of the ring-blockwise causal attention on
// tcgen05 tensor cores, all virtual ranks in persistent launches.
//
// The pages give only the backward of the all-to-all transpose ("LongVILA
// Guide", section "Implementation", UlyssesAllToAll.backward); the gradient
// of the attention itself is a reading: with P_ij = exp(s_ij - LSE_i)
// recomputed from the saved fp32 LSE and D_i = sum_d dO_i O_i,
//   dV_j = sum_i P_ij dO_i,  dS_ij = P_ij (dO_i . v_j - D_i),
//   dQ_i = scale sum_j dS_ij k_j,  dK_j = scale sum_i dS_ij q_i,
// dK, dV summed over the query heads of each kv head.
//
// Two kernels, so that no gradient is accumulated through global-memory
// reductions (a fused kernel adds a 64 KB dQ partial per (query tile, key
// tile) pair -- 15 TB at N = 512K -- and L2 reductions sustain only about
// 1.4 TB/s once the accumulator no longer fits in L2):
//
// attn_bwd_dkdv_kernel -- key-owner. Work unit: one kv head x one tile of
//   128 keys of one zigzag chunk; K, V stay in shared memory and dK, dV in
//   TMEM while the CTA visits every (query tile, query head) that sees the
//   keys, in ring order from the keys' side (at step s the block of rank k
//   sits on rank (k + s) mod P). Per visit: S^T = K Q^T, dP^T = V dO^T,
//   dV += P^T dO (A = P^T from TMEM), dK += dS^T Q.
// attn_bwd_dq_kernel -- query-owner, shaped like the forward. Work item:
//   one query head x 128 rows of one chunk; it visits its K/V tiles in ring
//   order with dQ accumulating in TMEM: S = Q K^T, dP = dO V^T, dQ += dS K.
//   dQ is written once per item (bf16, optionally fp32).
//
// Both: warp 0 TMA producer, warp 1 MMA issuer (warp-uniform, lane 0
// issues), warps 2-9 gradient warps, two per TMEM lane quarter, each
// thread owning one row and half (64) of the 128 columns. tcgen05 MMAs of
// one thread run in issue order, which the TMEM reuse below relies on.
#pragma once

#include <cuda.h>
#include <math_constants.h>

#include "ptx.cuh"
#include "ring.cuh"

namespace mmsp {
namespace bwd {

constexpr int BM = 128;               // rows of a tile (keys or queries)
constexpr int BN = 128;               // columns of a tile
constexpr int D = 128;                // head dim
constexpr int kThreads = 320;
constexpr int HALF = 128 * 128;       // bytes of a 128-row x 64-column bf16 half tile
constexpr int TILE = 128 * 128 * 2;   // 32 KB bf16 tile

struct Params {
  int32_t P, Hq, Hkv, G;
  int32_t rank_begin, n_ranks;  // virtual ranks of this launch: dQ of their queries, dK/dV of their keys
  int64_t C;        // chunk length
  int64_t Cp;       // chunk length padded to a multiple of 128 (LSE2/D rows)
  int32_t ntiles;   // 128-row tiles per chunk
  int32_t causal;
  int64_t n_units;  // dK/dV kernel work units
  int64_t n_items;  // dQ kernel work items
  float scale_log2;
  float scale;
  const float* lse2t;   // [P][Hq][2][Cp]: LSE * log2(e); +inf on padding
  const float* dt;      // [P][Hq][2][Cp]: D; 0 on padding
  __nv_bfloat16* dq;    // [N][Hq][d]
  float* dq_acc;        // [N][Hq][d] fp32 dQ or nullptr
  __nv_bfloat16* dk;    // [N][Hkv][d]
  __nv_bfloat16* dv;    // [N][Hkv][d]
  const int32_t* doc_start;  // [N] global order, first position of each token's document; or null
  long long wait_cap;
};

// Byte offset of 16-byte chunk `chunk16` (0..15) of `row` in a K-major,
// 128-byte-swizzled 128-row bf16 tile stored as two 64-column halves.
__device__ __forceinline__ uint32_t sw128(int row, int chunk16) {
  return (uint32_t)((chunk16 >> 3) * HALF + row * 128 + (((chunk16 & 7) ^ (row & 7)) << 4));
}

__device__ __forceinline__ void bulk_load_w(uint32_t leader, uint32_t dst, const void* src, uint32_t bytes,
                                            uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred q;\n\t"
      "setp.ne.b32 q, %4, 0;\n\t"
      "@q cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n\t}" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar), "r"(leader)
      : "memory");
}

// =========================================================== dK / dV kernel

struct Unit {
  int k, ck, kt, kvh;
  int64_t key0;  // first key of the tile within its chunk
  int gk;        // global chunk index of the keys
};

__device__ __forceinline__ Unit decode_unit(const Params& p, int64_t idx) {
  // groups of decreasing work over the launch's key ranks [b, b + n):
  // chunk 0 of rank b + g for g < n, then chunk 1 of rank b + 2n-1-g (the
  // whole ring visits global key chunk g as group g, chunk 0 first)
  const int64_t per_chunk = (int64_t)p.ntiles * p.Hkv;
  const int g = (int)(idx / per_chunk);
  const int64_t w = idx - (int64_t)g * per_chunk;
  Unit u;
  if (g < p.n_ranks) {
    u.k = p.rank_begin + g;
    u.ck = 0;
  } else {
    u.k = p.rank_begin + 2 * p.n_ranks - 1 - g;
    u.ck = 1;
  }
  u.gk = u.ck ? 2 * p.P - 1 - u.k : u.k;
  u.kvh = (int)(w / p.ntiles);
  u.kt = (int)(w % p.ntiles);
  u.key0 = (int64_t)u.kt * BM;
  return u;
}

// Enumerates the (query tile, head) visits of a unit in ring order. DOC:
// queries carry document bounds (packed sequences); compiled out otherwise.
template <bool DOC>
struct VisitIter {
  int k, P, gk, causal, G, kvh, s, qc, t, tmax, hg, ntiles;
  RingList ring;  // DOC: the few query chunks that can see the unit's keys
  int64_t C, key0, qrow_base, kg0, kg1, qchunk0;
  const int32_t* doc_start;
  bool in_chunk;
  int h, r, qcur;  // query head, rank, query chunk (0/1)
  int64_t q0;      // first query row of the tile within its chunk
  int64_t lrow0;   // first rank-local row of the tile
  int64_t qglob0;  // global position of the tile's first query
  bool diag;
  bool dmask;      // some query of the tile starts its document after a key of the unit

  __device__ __forceinline__ VisitIter(const Params& p, const Unit& u) {
    k = u.k;
    P = p.P;
    gk = u.gk;
    causal = p.causal;
    G = p.G;
    kvh = u.kvh;
    s = 0;
    qc = 0;
    t = 0;
    tmax = -1;
    hg = 0;
    ntiles = p.ntiles;
    C = p.C;
    key0 = u.key0;
    in_chunk = false;
    diag = false;
    dmask = false;
    doc_start = p.doc_start;
    kg0 = (int64_t)u.gk * p.C + u.key0;
    kg1 = (int64_t)u.gk * p.C + (u.key0 + BM - 1 < p.C - 1 ? u.key0 + BM - 1 : p.C - 1);
    ring.n = -1;
    if constexpr (DOC) {
      // queries see the keys only from chunk gk on, and only while their
      // document starts at or before the unit's last key: the visible query
      // chunks are [gk, c1] (document starts are non-decreasing). At step s
      // the keys' block sits on rank (k + s) mod P.
      int c1 = gk;
      while (c1 + 1 < 2 * P && c1 - gk < 4 && (int64_t)doc_start[(int64_t)(c1 + 1) * C] <= kg1) ++c1;
      ring.build(gk, c1, P, k, 1, 0, P);
    }
  }

  // Document test of the current query tile: false if every query's
  // document starts after the unit's last key (nothing visible).
  __device__ __forceinline__ bool doc_ok() {
    if constexpr (!DOC) return true;
    const int64_t qlast = qchunk0 + (q0 + BN - 1 < C - 1 ? q0 + BN - 1 : C - 1);
    if (doc_start[qglob0] > kg1) return false;
    dmask = doc_start[qlast] > kg0;
    return true;
  }

  __device__ __forceinline__ bool next() {
    while (true) {
      if (in_chunk) {
        if (hg < G) {
          h = kvh * G + hg;
          ++hg;
          return true;
        }
        hg = 0;
        ++t;
        while (t <= tmax) {
          q0 = (int64_t)t * BN;
          lrow0 = qrow_base + q0;
          qglob0 = qchunk0 + q0;
          if (doc_ok()) break;
          ++t;
        }
        if (t <= tmax) continue;
        in_chunk = false;
      }
      int sc;
      if (DOC && ring.n >= 0) {
        if (!ring.pop(sc, qcur)) return false;
      } else {
        if (s >= P) return false;
        sc = s;
        qcur = qc;
        if (++qc == 2) {
          qc = 0;
          ++s;
        }
      }
      r = (k + sc) % P;
      const int gq = qcur ? 2 * P - 1 - r : r;
      if (causal && gq < gk) continue;
      diag = causal && gq == gk;
      // diagonal: only query tiles that reach the tile's first key
      t = diag ? (int)(key0 / BN) : 0;
      tmax = ntiles - 1;
      hg = 0;
      qrow_base = (int64_t)r * 2 * C + (int64_t)qcur * C;
      qchunk0 = (int64_t)gq * C;
      while (t <= tmax) {
        q0 = (int64_t)t * BN;
        lrow0 = qrow_base + q0;
        qglob0 = qchunk0 + q0;
        if (doc_ok()) break;
        ++t;
      }
      in_chunk = t <= tmax;
    }
  }
};

struct SmemKV {
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = TILE;
  static constexpr int OFF_Q = 2 * TILE;   // two stages
  static constexpr int OFF_DO = 4 * TILE;  // two stages
  static constexpr int OFF_DST = 6 * TILE;
  static constexpr int OFF_VEC = 7 * TILE;  // two stages x (LSE2[128], D[128])
  static constexpr int OFF_BAR = OFF_VEC + 2 * 1024;
  static constexpr int NBAR = 20;
  static constexpr int BYTES = OFF_BAR + NBAR * 8 + 16;
  // Seven 32 KB tiles leave no room for alignment slack: the kernels need a
  // 1024-byte aligned dynamic shared memory base (it is, when a kernel has
  // no static shared memory) and report a layout error otherwise.
  static constexpr int ALLOC = BYTES;
};

template <bool DOC>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                         const __grid_constant__ Params p) {
  using L = SmemKV;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  if (base & 1023u) {
    if (threadIdx.x == 0) atomicExch(&g_timeout_flag, 2);
    return;
  }
  uint8_t* gbase = smem_raw;
  const uint32_t sK = base + L::OFF_K, sV = base + L::OFF_V;
  const uint32_t sQ0 = base + L::OFF_Q;
  const uint32_t sDO0 = base + L::OFF_DO;
  const uint32_t sDST = base + L::OFF_DST;
  const uint32_t sVEC = base + L::OFF_VEC;
  const float* vec_g = reinterpret_cast<const float*>(gbase + L::OFF_VEC);
  const uint32_t bar0 = base + L::OFF_BAR;
  const uint32_t kv_full = bar0, kv_empty = bar0 + 8;
  auto q_full = [&](int i) { return bar0 + 16u + 8u * i; };
  auto q_empty = [&](int i) { return bar0 + 32u + 8u * i; };
  auto do_full = [&](int i) { return bar0 + 48u + 8u * i; };
  auto do_empty = [&](int i) { return bar0 + 64u + 8u * i; };
  const uint32_t s_full = bar0 + 80, dp_full = bar0 + 88;
  const uint32_t p_full = bar0 + 96, dst_free = bar0 + 104;
  const uint32_t acc_full = bar0 + 112, acc_free = bar0 + 120;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::OFF_BAR + L::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::OFF_BAR + L::NBAR * 8 + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full(i), 1);
      mbar_init(q_empty(i), 1);
      mbar_init(do_full(i), 1);
      mbar_init(do_empty(i), 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 8);
    mbar_init(dst_free, 1);
    mbar_init(acc_full, 1);
    mbar_init(acc_free, 8);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const long long cap = p.wait_cap;
  // TMEM columns: S^T (then P^T as bf16 pairs: queries 0-63 in columns
  // [0,32), queries 64-127 in [64,96), each over S^T columns its own
  // writers have read), dP^T, dV, dK.
  const uint32_t cS = 0, cDP = 128, cDV = 256, cDK = 384;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    const uint32_t leader = lane == 0 ? 1u : 0u;
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
    }
    uint32_t ucnt = 0, vis = 0;
    for (int64_t idx = blockIdx.x; idx < p.n_units; idx += gridDim.x) {
      const Unit u = decode_unit(p, idx);
      if (ucnt > 0) mbar_wait(kv_empty, (ucnt - 1) & 1, abort_flag, cap);
      mbar_arrive_expect_tx_w(leader, kv_full, 2 * TILE);
      const int krow = (int)((int64_t)u.k * 2 * p.C + (int64_t)u.ck * p.C + u.key0);
      for (int hf = 0; hf < 2; ++hf) {
        tma_load_3d_w(leader, sK + hf * HALF, &tmK, kv_full, hf * 64, u.kvh, krow);
        tma_load_3d_w(leader, sV + hf * HALF, &tmV, kv_full, hf * 64, u.kvh, krow);
      }
      ++ucnt;
      VisitIter<DOC> it(p, u);
      while (it.next()) {
        const int st = vis & 1;
        const uint32_t use = vis >> 1;
        mbar_wait(q_empty(st), (use & 1) ^ 1, abort_flag, cap);
        mbar_arrive_expect_tx_w(leader, q_full(st), TILE + 1024);
        for (int hf = 0; hf < 2; ++hf)
          tma_load_3d_w(leader, sQ0 + st * TILE + hf * HALF, &tmQ, q_full(st), hf * 64, it.h, (int)it.lrow0);
        const int64_t vrow = (((int64_t)it.r * p.Hq + it.h) * 2 + it.qcur) * p.Cp + it.q0;
        bulk_load_w(leader, sVEC + st * 1024, p.lse2t + vrow, 512, q_full(st));
        bulk_load_w(leader, sVEC + st * 1024 + 512, p.dt + vrow, 512, q_full(st));
        mbar_wait(do_empty(st), (use & 1) ^ 1, abort_flag, cap);
        mbar_arrive_expect_tx_w(leader, do_full(st), TILE);
        for (int hf = 0; hf < 2; ++hf)
          tma_load_3d_w(leader, sDO0 + st * TILE + hf * HALF, &tmDO, do_full(st), hf * 64, it.h, (int)it.lrow0);
        ++vis;
      }
    }
    volatile int no_abort = 0;
    if (ucnt > 0) mbar_wait(kv_full, (ucnt - 1) & 1, &no_abort, cap);
    for (uint32_t i = (vis > 2 ? vis - 2 : 0); i < vis; ++i) {
      mbar_wait(q_full(i & 1), (i >> 1) & 1, &no_abort, cap);
      mbar_wait(do_full(i & 1), (i >> 1) & 1, &no_abort, cap);
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer
    // Once P^T_v (TMEM) and dS^T_v (smem) are ready: dV += P^T_v dO_v,
    // S^T_{v+1} (over P^T_v, after dV read it), dK += dS^T_v Q_v, dP^T_{v+1}.
    const uint32_t leader = lane == 0 ? 1u : 0u;
    constexpr uint32_t idKQ = idesc_bf16_f32(BM, BN, 0, 0);   // S^T, dP^T
    constexpr uint32_t idGrad = idesc_bf16_f32(BM, D, 0, 1);  // dV, dK: B MN-major
    const uint32_t tS = tmem + cS, tDP = tmem + cDP, tDV = tmem + cDV, tDK = tmem + cDK;
    uint32_t ucnt = 0, vis = 0, pc = 0, epi = 0;
    auto issue_kq = [&](uint32_t d_t, uint32_t a, uint32_t b) {  // d_t = a[128 x d] * b[128 x d]^T
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * HALF + (kk & 3) * 32;
        mma_bf16_ss_w(leader, d_t, desc_kmajor_sw128(a + off), desc_kmajor_sw128(b + off), idKQ, kk > 0 ? 1u : 0u);
      }
    };
    auto issue_s = [&](uint32_t v) {
      const int st = v & 1;
      mbar_wait(q_full(st), (v >> 1) & 1, abort_flag, cap);
      tc_fence_after();
      issue_kq(tS, sK, sQ0 + st * TILE);
      mma_commit_w(leader, s_full);
    };
    auto issue_dp = [&](uint32_t v) {
      const int st = v & 1;
      mbar_wait(do_full(st), (v >> 1) & 1, abort_flag, cap);
      tc_fence_after();
      issue_kq(tDP, sV, sDO0 + st * TILE);
      mma_commit_w(leader, dp_full);
    };
    for (int64_t idx = blockIdx.x; idx < p.n_units; idx += gridDim.x) {
      const Unit u = decode_unit(p, idx);
      mbar_wait(kv_full, ucnt & 1, abort_flag, cap);
      ++ucnt;
      tc_fence_after();
      VisitIter<DOC> it(p, u);
      bool has = it.next();
      bool first = true;
      if (has) {
        issue_s(vis);
        issue_dp(vis);
      }
      while (has) {
        const int st = vis & 1;
        mbar_wait(p_full, pc & 1, abort_flag, cap);
        ++pc;
        tc_fence_after();
        if (first && epi > 0) {
          mbar_wait(acc_free, (epi - 1) & 1, abort_flag, cap);
          tc_fence_after();
        }
        // dV += P^T dO: A = P^T from TMEM (8 columns = 16 queries per step)
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_bf16_ts_w(leader, tDV, tS + (uint32_t)((kk >> 2) * 64 + (kk & 3) * 8),
                        desc_mnmajor_sw128(sDO0 + st * TILE + kk * 2048, HALF), idGrad,
                        (kk > 0 || !first) ? 1u : 0u);
        mma_commit_w(leader, do_empty(st));
        has = it.next();
        if (has) issue_s(vis + 1);
        // dK += dS^T Q
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * HALF + (kk & 3) * 32;
          mma_bf16_ss_w(leader, tDK, desc_kmajor_sw128(sDST + aoff),
                        desc_mnmajor_sw128(sQ0 + st * TILE + kk * 2048, HALF), idGrad,
                        (kk > 0 || !first) ? 1u : 0u);
        }
        mma_commit_w(leader, q_empty(st));
        mma_commit_w(leader, dst_free);
        if (has) issue_dp(vis + 1);
        ++vis;
        first = false;
      }
      mma_commit_w(leader, kv_empty);
      mma_commit_w(leader, acc_full);
      ++epi;
    }
  } else {
    // ------------------------------------------- gradient rows (8 warps)
    const int grp = (warp - 2) >> 2;  // which 64 of the 128 query columns
    const int wq = warp & 3;
    const int row = wq * 32 + lane;  // key within the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + cS + lane_off;
    const uint32_t tDP = tmem + cDP + lane_off;
    const uint32_t cq = 64u * grp;  // this thread's first query column
    const float sl2 = p.scale_log2;
    uint32_t vis = 0, sc = 0, dpc = 0, dstc = 0, accc = 0;
    for (int64_t idx = blockIdx.x; idx < p.n_units; idx += gridDim.x) {
      const Unit u = decode_unit(p, idx);
      const int64_t kin = u.key0 + row;  // key index within its chunk
      const bool key_ok = kin < p.C;
      VisitIter<DOC> it(p, u);
      while (it.next()) {
        const int st = vis & 1;
        const float* lse2 = vec_g + st * 256;
        const float* dvec = lse2 + 128;
        // visible query columns: c >= cmin (diagonal); none for keys past C
        int cmin = 0, cmax = 128;  // visible query columns [cmin, cmax)
        if (!key_ok) cmin = 128;
        else if (it.diag) {
          const int64_t dmin = kin - it.q0;
          cmin = dmin <= 0 ? 0 : (dmin >= 128 ? 128 : (int)dmin);
        }
        if (DOC && it.dmask && key_ok) {
          // first column whose document starts after this key (document
          // starts are non-decreasing along the queries): binary search
          const int64_t gkey = it.kg0 + row;
          int lo = 0, hi = (int)(p.C - it.q0 < 128 ? p.C - it.q0 : 128);
          while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if ((int64_t)p.doc_start[it.qglob0 + mid] > gkey) hi = mid;
            else lo = mid + 1;
          }
          cmax = lo;
        }
        mbar_wait(q_full(st), (vis >> 1) & 1, abort_flag, cap);  // LSE2/D arrive with Q
        // S^T -> P^T, written back as bf16 pairs over read columns
        mbar_wait(s_full, sc & 1, abort_flag, cap);
        ++sc;
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t sr[32];
          tmem_ld32(tS + cq + 32u * h, sr);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const int c = (int)cq + 32 * h + j;
            const float4 lv = *reinterpret_cast<const float4*>(lse2 + c);
            float e0 = ex2_approx(fmaf(__uint_as_float(sr[j]), sl2, -lv.x));
            float e1 = ex2_approx(fmaf(__uint_as_float(sr[j + 1]), sl2, -lv.y));
            float e2 = ex2_approx(fmaf(__uint_as_float(sr[j + 2]), sl2, -lv.z));
            float e3 = ex2_approx(fmaf(__uint_as_float(sr[j + 3]), sl2, -lv.w));
            if (c < cmin || c >= cmax) e0 = 0.f;
            if (c + 1 < cmin || c + 1 >= cmax) e1 = 0.f;
            if (c + 2 < cmin || c + 2 >= cmax) e2 = 0.f;
            if (c + 3 < cmin || c + 3 >= cmax) e3 = 0.f;
            pk[j / 2] = pack_bf16x2(e0, e1);
            pk[j / 2 + 1] = pack_bf16x2(e2, e3);
          }
          tmem_st16(tS + cq + 16u * h, pk);
        }
        tmem_wait_st();
        // dP^T -> dS^T = P^T (dP^T - D) into shared memory, once the dK MMA
        // of the previous visit no longer reads it
        mbar_wait(dp_full, dpc & 1, abort_flag, cap);
        ++dpc;
        tc_fence_after();
        if (dstc < vis) {
          mbar_wait(dst_free, dstc & 1, abort_flag, cap);
          ++dstc;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t sr[32];
          uint32_t pv[16];
          tmem_ld32(tDP + cq + 32u * h, sr);
          tmem_ld16(tS + cq + 16u * h, pv);
          tmem_wait_ld();
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            const int c0 = (int)cq + 32 * h + 8 * c8;  // first query of this 16-byte chunk
            const float4 dv0 = *reinterpret_cast<const float4*>(dvec + c0);
            const float4 dv1 = *reinterpret_cast<const float4*>(dvec + c0 + 4);
            const float dd[8] = {dv0.x, dv0.y, dv0.z, dv0.w, dv1.x, dv1.y, dv1.z, dv1.w};
            uint32_t o[4];
#pragma unroll
            for (int u2 = 0; u2 < 4; ++u2) {
              const int j = 8 * c8 + 2 * u2;
              const __nv_bfloat162 pp = *reinterpret_cast<const __nv_bfloat162*>(&pv[4 * c8 + u2]);
              const float d0 = __low2float(pp) * (__uint_as_float(sr[j]) - dd[2 * u2]);
              const float d1 = __high2float(pp) * (__uint_as_float(sr[j + 1]) - dd[2 * u2 + 1]);
              o[u2] = pack_bf16x2(d0, d1);
            }
            st_shared_v4(sDST + sw128(row, c0 / 8), o[0], o[1], o[2], o[3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        ++vis;
      }
      // unit epilogue: this thread's 64 columns of dV and dK (dK scaled)
      mbar_wait(acc_full, accc & 1, abort_flag, cap);
      ++accc;
      tc_fence_after();
      const int64_t krow = (int64_t)u.k * 2 * p.C + (int64_t)u.ck * p.C + kin;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const uint32_t tA = tmem + (which ? cDK : cDV) + lane_off + cq;
        __nv_bfloat16* out = which ? p.dk : p.dv;
        const float f = which ? p.scale : 1.f;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t a[32];
          tmem_ld32(tA + 32u * c, a);
          tmem_wait_ld();
          if (key_ok) {
            uint4* dst = reinterpret_cast<uint4*>(out + (krow * p.Hkv + u.kvh) * D + cq + 32 * c);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_uint4(pack_bf16x2(__uint_as_float(a[8 * j]) * f, __uint_as_float(a[8 * j + 1]) * f),
                                  pack_bf16x2(__uint_as_float(a[8 * j + 2]) * f, __uint_as_float(a[8 * j + 3]) * f),
                                  pack_bf16x2(__uint_as_float(a[8 * j + 4]) * f, __uint_as_float(a[8 * j + 5]) * f),
                                  pack_bf16x2(__uint_as_float(a[8 * j + 6]) * f, __uint_as_float(a[8 * j + 7]) * f));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_free);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ================================================================ dQ kernel

struct QItem {
  int r, c, t, h, kvh;
  int64_t q0;     // first query row of the tile within its chunk
  int64_t lrow0;  // first rank-local row
};

__device__ __forceinline__ QItem decode_qitem(const Params& p, int64_t idx) {
  // groups of decreasing work over the launch's query ranks [b, b + n):
  // chunk 1 of rank b + g for g < n, then chunk 0 of rank b + 2n-1-g (the
  // whole ring visits global query chunk 2P-1-g as group g)
  const int64_t per_group = (int64_t)p.ntiles * p.Hq;
  const int g = (int)(idx / per_group);
  const int64_t w = idx - (int64_t)g * per_group;
  QItem it;
  if (g < p.n_ranks) {
    it.r = p.rank_begin + g;
    it.c = 1;
  } else {
    it.r = p.rank_begin + 2 * p.n_ranks - 1 - g;
    it.c = 0;
  }
  const int hg = (int)(w % p.G);
  const int64_t w2 = w / p.G;
  it.t = (int)(w2 % p.ntiles);
  it.kvh = (int)(w2 / p.ntiles);
  it.h = it.kvh * p.G + hg;
  it.q0 = (int64_t)it.t * BM;
  it.lrow0 = (int64_t)it.r * 2 * p.C + (int64_t)it.c * p.C + it.q0;
  return it;
}

// K/V tiles a query tile visits, in ring order (rank r holds rank (r-s)
// mod P's block at step s).
template <bool DOC>
struct KVIter {
  int r, P, gq, causal, s, ck, t, tmax, ntiles;
  RingList ring;  // DOC: the few chunks that can hold visible keys
  int64_t C, q0, base_row, kchunk0, lo_min, lo_max;
  bool in_chunk, diag;
  int64_t kv_row, kglob0;
  int key0;
  bool mask;

  __device__ __forceinline__ KVIter(const Params& p, const QItem& it) {
    r = it.r;
    P = p.P;
    gq = it.c ? 2 * p.P - 1 - it.r : it.r;
    causal = p.causal;
    s = 0;
    ck = 0;
    t = 0;
    tmax = -1;
    ntiles = p.ntiles;
    C = p.C;
    q0 = it.q0;
    in_chunk = false;
    diag = false;
    lo_min = lo_max = 0;
    if constexpr (DOC) {
      const int64_t g0 = (int64_t)gq * C;
      lo_min = p.doc_start[g0 + q0];
      lo_max = p.doc_start[g0 + (q0 + BM - 1 < C - 1 ? q0 + BM - 1 : C - 1)];
      // only chunks [lo_min / C, gq] can hold visible keys; at step s the
      // rank holds the K/V of rank (r - s) mod P
      ring.build((int)(lo_min / C), gq, P, r, -1, 0, P);
    } else {
      ring.n = -1;
    }
  }

  __device__ __forceinline__ bool next() {
    while (true) {
      if (!in_chunk) {
        int sc, ckc;
        if (DOC && ring.n >= 0) {
          if (!ring.pop(sc, ckc)) return false;
        } else {
          if (s >= P) return false;
          sc = s;
          ckc = ck;
          if (++ck == 2) {
            ck = 0;
            ++s;
          }
        }
        int k = (r - sc) % P;
        if (k < 0) k += P;
        const int gk = ckc ? 2 * P - 1 - k : k;
        const bool skip = causal && gk > gq;
        diag = causal && gk == gq;
        base_row = (int64_t)k * 2 * C + (int64_t)ckc * C;
        kchunk0 = (int64_t)gk * C;
        if (skip) continue;
        if (DOC && kchunk0 + C - 1 < lo_min) continue;  // whole chunk before every document
        int64_t last = q0 + BM - 1;
        if (last > C - 1) last = C - 1;
        tmax = diag ? (int)(last / BN) : ntiles - 1;
        // tiles wholly before every row's document hold no visible key
        t = (DOC && lo_min > kchunk0) ? (int)((lo_min - kchunk0) / BN) : 0;
        in_chunk = true;
      }
      if (t > tmax) {
        in_chunk = false;
        continue;
      }
      key0 = t * BN;
      ++t;
      kglob0 = kchunk0 + key0;
      const int64_t klast = kchunk0 + ((int64_t)key0 + BN - 1 < C - 1 ? (int64_t)key0 + BN - 1 : C - 1);
      if (DOC && klast < lo_min) continue;
      mask = (diag && (int64_t)key0 + BN - 1 > q0) || ((int64_t)key0 + BN > C) || (DOC && kglob0 < lo_max);
      kv_row = base_row + key0;
      return true;
    }
  }
};

struct SmemQ {
  static constexpr int NK = 3;  // K ring stages (K_j is read by S(j) and dQ(j))
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = TILE;
  static constexpr int OFF_DS = 2 * TILE;
  static constexpr int OFF_K = 3 * TILE;
  static constexpr int OFF_V = OFF_K + NK * TILE;  // one V stage (read by dP(j) only)
  static constexpr int OFF_BAR = OFF_V + TILE;
  static constexpr int NBAR = 2 * NK + 14;
  static constexpr int BYTES = OFF_BAR + NBAR * 8 + 16;
  static constexpr int ALLOC = BYTES;  // needs a 1024-aligned base (see SmemKV)
};

template <bool DOC>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                       const __grid_constant__ Params p) {
  using L = SmemQ;
  constexpr int NK = L::NK;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  if (base & 1023u) {
    if (threadIdx.x == 0) atomicExch(&g_timeout_flag, 2);
    return;
  }
  uint8_t* gbase = smem_raw;
  const uint32_t sQ = base + L::OFF_Q, sDO = base + L::OFF_DO, sDS = base + L::OFF_DS;
  const uint32_t sK0 = base + L::OFF_K, sV = base + L::OFF_V;
  const uint32_t bar0 = base + L::OFF_BAR;
  auto k_full = [&](int i) { return bar0 + 8u * i; };
  auto k_empty = [&](int i) { return bar0 + 8u * (NK + i); };
  const uint32_t v_full = bar0 + 8u * (2 * NK), v_empty = v_full + 8;
  const uint32_t q_full = v_full + 16, q_empty = v_full + 24;
  auto s_full = [&](int b) { return v_full + 32u + 8u * b; };
  auto s_free = [&](int b) { return v_full + 48u + 8u * b; };
  const uint32_t dp_full = v_full + 64, ds_full = v_full + 72, ds_free = v_full + 80;
  const uint32_t dq_done = v_full + 88, dq_free = v_full + 96;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::OFF_BAR + L::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::OFF_BAR + L::NBAR * 8 + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NK; ++i) {
      mbar_init(k_full(i), 1);
      mbar_init(k_empty(i), 1);
    }
    mbar_init(v_full, 1);
    mbar_init(v_empty, 1);
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full(b), 1);
      mbar_init(s_free(b), 8);
    }
    mbar_init(dp_full, 1);
    mbar_init(ds_full, 8);
    mbar_init(ds_free, 1);
    mbar_init(dq_done, 1);
    mbar_init(dq_free, 8);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const long long cap = p.wait_cap;
  // TMEM columns: S buffers 0 and 1, dP, dQ.
  const uint32_t cS0 = 0, cDP = 256, cDQ = 384;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    const uint32_t leader = lane == 0 ? 1u : 0u;
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
    }
    uint32_t icnt = 0, kc = 0, vc = 0;
    for (int64_t idx = blockIdx.x; idx < p.n_items; idx += gridDim.x) {
      const QItem it = decode_qitem(p, idx);
      if (icnt > 0) mbar_wait(q_empty, (icnt - 1) & 1, abort_flag, cap);
      mbar_arrive_expect_tx_w(leader, q_full, 2 * TILE);
      for (int hf = 0; hf < 2; ++hf) {
        tma_load_3d_w(leader, sQ + hf * HALF, &tmQ, q_full, hf * 64, it.h, (int)it.lrow0);
        tma_load_3d_w(leader, sDO + hf * HALF, &tmDO, q_full, hf * 64, it.h, (int)it.lrow0);
      }
      ++icnt;
      KVIter<DOC> ki(p, it);
      while (ki.next()) {
        const int st = (int)(kc % NK);
        mbar_wait(k_empty(st), ((kc / NK) & 1) ^ 1, abort_flag, cap);
        mbar_arrive_expect_tx_w(leader, k_full(st), TILE);
        for (int hf = 0; hf < 2; ++hf)
          tma_load_3d_w(leader, sK0 + st * TILE + hf * HALF, &tmK, k_full(st), hf * 64, it.kvh, (int)ki.kv_row);
        ++kc;
        mbar_wait(v_empty, (vc & 1) ^ 1, abort_flag, cap);
        mbar_arrive_expect_tx_w(leader, v_full, TILE);
        for (int hf = 0; hf < 2; ++hf)
          tma_load_3d_w(leader, sV + hf * HALF, &tmV, v_full, hf * 64, it.kvh, (int)ki.kv_row);
        ++vc;
      }
    }
    volatile int no_abort = 0;
    for (uint32_t i = (kc > NK ? kc - NK : 0); i < kc; ++i)
      mbar_wait(k_full((int)(i % NK)), (i / NK) & 1, &no_abort, cap);
    if (vc > 0) mbar_wait(v_full, (vc - 1) & 1, &no_abort, cap);
    if (icnt > 0) mbar_wait(q_full, (icnt - 1) & 1, &no_abort, cap);
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer
    // Per K/V tile j: S(j+1) into the other S buffer ahead of time; once
    // dS(j) is in shared memory, dQ += dS(j) K_j, then dP(j+1).
    const uint32_t leader = lane == 0 ? 1u : 0u;
    constexpr uint32_t idS = idesc_bf16_f32(BM, BN, 0, 0);
    constexpr uint32_t idDQ = idesc_bf16_f32(BM, D, 0, 1);  // B = K read MN-major
    const uint32_t tDP = tmem + cDP, tDQ = tmem + cDQ;
    uint32_t icnt = 0, kc = 0, vc = 0, scnt = 0, dsc = 0, epi = 0;
    uint32_t sfree_cnt[2] = {0, 0};
    auto issue_qk = [&](uint32_t d_t, uint32_t a, uint32_t b) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * HALF + (kk & 3) * 32;
        mma_bf16_ss_w(leader, d_t, desc_kmajor_sw128(a + off), desc_kmajor_sw128(b + off), idS, kk > 0 ? 1u : 0u);
      }
    };
    // S of K tile number k (ring stage k % NK) into S buffer scnt & 1, once
    // the gradient warps have read that buffer's previous tile
    auto issue_s = [&](uint32_t k) {
      const int b = scnt & 1;
      if (scnt >= 2) {
        mbar_wait(s_free(b), sfree_cnt[b] & 1, abort_flag, cap);
        ++sfree_cnt[b];
        tc_fence_after();
      }
      mbar_wait(k_full((int)(k % NK)), (k / NK) & 1, abort_flag, cap);
      tc_fence_after();
      issue_qk(tmem + cS0 + 128u * b, sQ, sK0 + (k % NK) * TILE);
      mma_commit_w(leader, s_full(b));
      ++scnt;
    };
    auto issue_dp = [&]() {
      mbar_wait(v_full, vc & 1, abort_flag, cap);
      tc_fence_after();
      issue_qk(tDP, sDO, sV);
      mma_commit_w(leader, dp_full);
      mma_commit_w(leader, v_empty);
      ++vc;
    };
    for (int64_t idx = blockIdx.x; idx < p.n_items; idx += gridDim.x) {
      const QItem it = decode_qitem(p, idx);
      mbar_wait(q_full, icnt & 1, abort_flag, cap);
      ++icnt;
      tc_fence_after();
      KVIter<DOC> ki(p, it);
      bool has = ki.next();
      uint32_t kcur = kc;
      if (has) {
        issue_s(kc++);
        issue_dp();
      }
      bool first = true;
      while (has) {
        const bool has_next = ki.next();
        uint32_t knext = 0;
        if (has_next) {
          knext = kc++;
          issue_s(knext);
        }
        // dS(j) ready in shared memory (and dP(j) read)
        mbar_wait(ds_full, dsc & 1, abort_flag, cap);
        ++dsc;
        tc_fence_after();
        if (first && epi > 0) {
          mbar_wait(dq_free, (epi - 1) & 1, abort_flag, cap);
          tc_fence_after();
        }
        const uint32_t sk = sK0 + (kcur % NK) * TILE;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * HALF + (kk & 3) * 32;
          mma_bf16_ss_w(leader, tDQ, desc_kmajor_sw128(sDS + aoff), desc_mnmajor_sw128(sk + kk * 2048, HALF), idDQ,
                        (kk > 0 || !first) ? 1u : 0u);
        }
        mma_commit_w(leader, ds_free);
        mma_commit_w(leader, k_empty((int)(kcur % NK)));
        if (has_next) issue_dp();
        first = false;
        has = has_next;
        kcur = knext;
      }
      mma_commit_w(leader, q_empty);
      if (!first) {
        mma_commit_w(leader, dq_done);
        ++epi;
      }
    }
  } else {
    // ------------------------------------------- gradient rows (8 warps)
    const int grp = (warp - 2) >> 2;  // which 64 of the 128 key columns
    const int wq = warp & 3;
    const int row = wq * 32 + lane;  // query row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t cq = 64u * grp;
    const float sl2 = p.scale_log2;
    uint32_t scnt = 0, tiles = 0, icnt = 0;
    for (int64_t idx = blockIdx.x; idx < p.n_items; idx += gridDim.x) {
      const QItem it = decode_qitem(p, idx);
      const int64_t qin = it.q0 + row;  // query row within its chunk
      // this row's LSE*log2(e) and D (padding rows: +inf and 0)
      const int64_t vrow = (((int64_t)it.r * p.Hq + it.h) * 2 + it.c) * p.Cp + qin;
      const float lse2 = p.lse2t[vrow];
      const float dval = p.dt[vrow];
      const int64_t gq_row = (int64_t)(it.c ? 2 * p.P - 1 - it.r : it.r) * p.C + qin;
      const int64_t lo_row = (DOC && qin < p.C) ? (int64_t)p.doc_start[gq_row] : 0;
      KVIter<DOC> ki(p, it);
      bool any = false;
      while (ki.next()) {
        any = true;
        int lim = 128, lb = 0;  // visible key columns of this row in the tile: [lb, lim)
        if (ki.mask) {
          int64_t l = p.C - ki.key0;
          if (ki.diag) {
            const int64_t dl = qin - ki.key0 + 1;
            l = dl < l ? dl : l;
          }
          lim = l < 0 ? 0 : (l > 128 ? 128 : (int)l);
          if (DOC) {
            const int64_t b = lo_row - ki.kglob0;
            lb = b < 0 ? 0 : (b > 128 ? 128 : (int)b);
          }
        }
        const int b = scnt & 1;
        mbar_wait(s_full(b), (scnt >> 1) & 1, abort_flag, cap);
        ++scnt;
        tc_fence_after();
        uint32_t pk[32];  // P as bf16 pairs for this thread's 64 key columns
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t sr[32];
          tmem_ld32(tmem + cS0 + 128u * b + lane_off + cq + 32u * h, sr);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const int c = (int)cq + 32 * h + j;
            float e0 = ex2_approx(fmaf(__uint_as_float(sr[j]), sl2, -lse2));
            float e1 = ex2_approx(fmaf(__uint_as_float(sr[j + 1]), sl2, -lse2));
            if (c >= lim || c < lb) e0 = 0.f;
            if (c + 1 >= lim || c + 1 < lb) e1 = 0.f;
            pk[16 * h + j / 2] = pack_bf16x2(e0, e1);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free(b));
        mbar_wait(dp_full, tiles & 1, abort_flag, cap);
        tc_fence_after();
        // the dS buffer is free once the previous tile's dQ MMA read it
        if (tiles > 0) mbar_wait(ds_free, (tiles - 1) & 1, abort_flag, cap);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t sr[32];
          tmem_ld32(tmem + cDP + lane_off + cq + 32u * h, sr);
          tmem_wait_ld();
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            uint32_t o[4];
#pragma unroll
            for (int u2 = 0; u2 < 4; ++u2) {
              const int j = 8 * c8 + 2 * u2;
              const __nv_bfloat162 pp = *reinterpret_cast<const __nv_bfloat162*>(&pk[16 * h + j / 2]);
              const float d0 = __low2float(pp) * (__uint_as_float(sr[j]) - dval);
              const float d1 = __high2float(pp) * (__uint_as_float(sr[j + 1]) - dval);
              o[u2] = pack_bf16x2(d0, d1);
            }
            st_shared_v4(sDS + sw128(row, (int)(cq / 8) + 4 * h + c8), o[0], o[1], o[2], o[3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_full);
        ++tiles;
      }
      // item epilogue: dQ = scale * accumulator, this thread's 64 columns
      if (any) {
        mbar_wait(dq_done, icnt & 1, abort_flag, cap);
        ++icnt;
        tc_fence_after();
      }
      const bool row_ok = qin < p.C;
      const int64_t rh = (it.lrow0 + row) * p.Hq + it.h;
      const float sc = p.scale;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t a[32];
        if (any) {
          tmem_ld32(tmem + cDQ + lane_off + cq + 32u * c, a);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) a[j] = 0u;
        }
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(p.dq + rh * D + cq + 32 * c);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[j] = make_uint4(pack_bf16x2(__uint_as_float(a[8 * j]) * sc, __uint_as_float(a[8 * j + 1]) * sc),
                                pack_bf16x2(__uint_as_float(a[8 * j + 2]) * sc, __uint_as_float(a[8 * j + 3]) * sc),
                                pack_bf16x2(__uint_as_float(a[8 * j + 4]) * sc, __uint_as_float(a[8 * j + 5]) * sc),
                                pack_bf16x2(__uint_as_float(a[8 * j + 6]) * sc, __uint_as_float(a[8 * j + 7]) * sc));
          if (p.dq_acc) {
            float4* d32 = reinterpret_cast<float4*>(p.dq_acc + rh * D + cq + 32 * c);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              d32[j] = make_float4(__uint_as_float(a[4 * j]) * sc, __uint_as_float(a[4 * j + 1]) * sc,
                                   __uint_as_float(a[4 * j + 2]) * sc, __uint_as_float(a[4 * j + 3]) * sc);
          }
        }
      }
      if (any) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dq_free);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// D_i = sum_d dO_i * O_i (fp32) and LSE_i * log2(e), written per head into
// the padded, rank-major [P][Hq][2][Cp] layout (+inf / 0 on padding rows),
// for the rows of virtual ranks [rank_begin, rank_begin + n_ranks) (each
// rank's rows are one contiguous slab, so a GPU that owns a range of ranks
// can exchange its slab whole). One warp per (row, head); 8-byte loads.
__global__ void __launch_bounds__(256) bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                      const __nv_bfloat16* __restrict__ dout,
                                                      const float* __restrict__ lse, float* __restrict__ lse2t,
                                                      float* __restrict__ dt, int32_t rank_begin, int32_t n_ranks,
                                                      int32_t Hq, int64_t C, int64_t Cp) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t total = (int64_t)n_ranks * 2 * Cp * Hq;  // padded (row, head) pairs of the launch's ranks
  for (int64_t w = warp; w < total; w += nwarps) {
    const int h = (int)(w % Hq);
    const int64_t pr = w / Hq;   // padded row within the range: (r'*2 + c)*Cp + t
    const int64_t t = pr % Cp;
    const int64_t rc = pr / Cp + 2 * (int64_t)rank_begin;  // r*2 + c
    const int64_t out_idx = (((rc >> 1) * Hq + h) * 2 + (rc & 1)) * Cp + t;
    if (t >= C) {
      if (lane == 0) {
        lse2t[out_idx] = CUDART_INF_F;
        dt[out_idx] = 0.f;
      }
      continue;
    }
    const int64_t lrow = rc * C + t;
    const int64_t rh = lrow * Hq + h;
    const uint2 a = reinterpret_cast<const uint2*>(o + rh * D)[lane];
    const uint2 b = reinterpret_cast<const uint2*>(dout + rh * D)[lane];
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
    float s = __low2float(a2[0]) * __low2float(b2[0]) + __high2float(a2[0]) * __high2float(b2[0]) +
              __low2float(a2[1]) * __low2float(b2[1]) + __high2float(a2[1]) * __high2float(b2[1]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) {
      lse2t[out_idx] = lse[rh] * 1.4426950408889634f;
      dt[out_idx] = s;
    }
  }
}

}  // namespace bwd
}  // namespace mmsp
