// attn_fwd.cuh -- ring-blockwise causal attention forward on tcgen05 tensor
// cores, all P virtual ranks of the ring in one persistent launch.
//
// Method: "LongVILA Guide" (aifetchly), section "Implementation",
// LongVILAMultiModalAttention.forward: for ring_size steps each rank runs
// block attention of its queries against the K/V block it currently holds
// (scores scaled by 1/sqrt(head_dim)), then receives the next block from the
// previous ring rank (LongVILAParallelContext, "Identify Ring Neighbors").
// So rank r holds the K/V of rank (r - s) mod P at step s. The per-step
// results are merged with the online-softmax (log-sum-exp) combine -- a
// reading; the page's sketch sums normalised blocks -- which, carried in
// registers/TMEM across the steps, is the fused form of mmsp_lse_merge.
//
// Work unit ("item"): one head h and 256 consecutive query rows (two 128-row
// tiles A and B) of one zigzag chunk of one virtual rank. Items are ordered
// by decreasing causal work (q chunk 2P-1 first), then kv head, row block,
// query head, so CTAs running together stream the same K/V tiles through L2.
// A launch may cover a range of virtual ranks only (the ranks one GPU owns
// when the ring is split across GPUs); it reads every rank's K/V.
// The CTA visits the item's K/V tiles of 128 keys in ring order and skips
// (chunk, tile) pairs the causal mask empties.
//
// Warp roles (384 threads = three warpgroups, one CTA per SM):
//   warp 0      TMA producer: Q tiles A/B once per item, then K_j, V_j into
//               a 5-stage ring of 128 x d bf16 tiles (128-byte swizzle).
//   warp 1      MMA issuer for tile A, warp 2 for tile B (warp-uniform, one
//               lane issues): S_X = Q_X K_j^T into TMEM, and O_X += P_X V_j
//               with P_X read from TMEM (the softmax writes bf16 P over the
//               S columns it has consumed), in the order PV_X(j), S_X(j+1),
//               so the tensor core works on one tile while the softmax warps
//               work on the other. tcgen05 MMAs of one thread run in issue
//               order, so S_X(j+1) overwrites P_X(j) only after PV_X(j) read
//               it. Without document masks an issue token (two named
//               barriers) keeps the tiles' groups in the order A, B per step.
//   warp 3      idle (it completes the first warpgroup's register release).
//   warps 4-7   softmax for tile A, warps 8-11 for tile B: one thread per
//               row (TMEM lane) holding its whole row of S in registers,
//               fp32 online softmax in base 2, P written to TMEM as bf16,
//               the running max raised (and O rescaled) whenever a tile
//               holds a larger score (with documents: past a 2^8 margin,
//               the dominant term of O corrected in the epilogue),
//               epilogue O / l and LSE.
// The first warpgroup gives registers to the two softmax warpgroups
// (setmaxnreg), see kRegCtl / kRegSoftmax.
// TMEM: S_A [0,128) S_B [128,256) O_A [256,256+d) O_B [256+d,256+2d).
#pragma once

#include <cuda.h>
#include <math_constants.h>

#include <type_traits>

#include "ptx.cuh"
#include "ring.cuh"

namespace mmsp {
namespace fwd {

constexpr int BM = 128;      // query rows per tile
constexpr int BN = 128;      // keys per tile
constexpr int NSTAGE = 5;    // K/V ring stages
constexpr int kThreads = 384;  // three warpgroups: TMA + 2 MMA (+1 idle warp), softmax A, softmax B
// Register split: the launch gives 168 per thread (384 x 168 <= 65,536);
// the control warpgroup drops to kRegCtl and the softmax warpgroups rise to
// kRegSoftmax, keeping 128 x kRegCtl + 256 x kRegSoftmax <= 384 x 168.
constexpr int kRegLaunch = 168;
constexpr int kRegCtl = 120;
constexpr int kRegSoftmax = 176;
static_assert(128 * kRegCtl + 256 * kRegSoftmax <= kThreads * kRegLaunch, "register split exceeds the launch");
constexpr int HALF = 128 * 128;  // bytes of one 128-row x 64-column bf16 half tile

struct Params {
  int32_t P, Hq, Hkv, G;
  int32_t rank_begin, n_ranks;  // the virtual ranks this launch computes: [rank_begin, rank_begin + n_ranks)
  int64_t C;        // zigzag chunk length N / (2P)
  int32_t nblk;     // 256-row blocks per chunk
  int32_t causal, step_begin, step_end;
  int32_t accumulate, finalize;
  int64_t n_items;
  float scale_log2;  // softmax scale * log2(e)
  float* o_acc;
  float* lse;
  __nv_bfloat16* o_out;
  const int32_t* doc_start;  // [N] global order, first position of each token's document; or null
  long long wait_cap;
};

struct Item {
  int r, c, blk, h, kvh;
  int64_t rowA0;       // first row of tile A within its chunk
  bool validA, validB;
};

__device__ __forceinline__ Item decode_item(const Params& p, int64_t idx) {
  const int64_t per_group = (int64_t)p.nblk * p.Hq;
  const int g = (int)(idx / per_group);
  const int64_t w = idx - (int64_t)g * per_group;
  Item it;
  // groups in decreasing causal work over the launch's ranks [b, b + n):
  // chunk 1 of rank b + g (global chunk 2P-1-b-g) for g < n, then chunk 0
  // of rank b + 2n-1-g (global chunk b + 2n-1-g). The whole ring (b = 0,
  // n = P) visits global query chunk 2P-1-g as group g.
  if (g < p.n_ranks) {
    it.r = p.rank_begin + g;
    it.c = 1;
  } else {
    it.r = p.rank_begin + 2 * p.n_ranks - 1 - g;
    it.c = 0;
  }
  const int hg = (int)(w % p.G);
  const int64_t w2 = w / p.G;
  it.blk = (int)(w2 % p.nblk);
  it.kvh = (int)(w2 / p.nblk);
  it.h = it.kvh * p.G + hg;
  it.rowA0 = (int64_t)it.blk * 256;
  it.validA = it.rowA0 < p.C;
  it.validB = it.rowA0 + 128 < p.C;
  return it;
}

// Enumerates the K/V tiles an item visits, in ring order. DOC: rows carry
// document bounds (packed sequences); compiled out otherwise.
template <bool DOC>
struct TileIter {
  int r, P, gq, causal, s, se, ck, t, tmax, ntiles;
  RingList ring;  // DOC: the few chunks that can hold visible keys
  int64_t C, rowA0, base_row;
  int32_t kchunk0;  // global position of the current K/V chunk (N < 2^31)
  bool validA, validB, in_chunk, diag;
  // document bounds (global positions): the smallest and largest first key
  // position over the rows of tiles A and B (0 without documents)
  int32_t loA_min, loA_max, loB_min, loB_max;
  // current tile
  int64_t kv_row;
  int32_t kglob0;
  int key0;
  bool actA, actB, maskA, maskB;

  __device__ __forceinline__ TileIter(const Params& p, const Item& it) {
    r = it.r;
    P = p.P;
    gq = it.c ? 2 * p.P - 1 - it.r : it.r;
    causal = p.causal;
    s = p.step_begin;
    se = p.step_end;
    ck = 0;
    t = 0;
    tmax = -1;
    C = p.C;
    ntiles = (int)((p.C + BN - 1) / BN);
    rowA0 = it.rowA0;
    validA = it.validA;
    validB = it.validB;
    in_chunk = false;
    diag = false;
    loA_min = loA_max = loB_min = loB_max = 0;
    if constexpr (DOC) {
      const int32_t g0 = gq * (int32_t)C;
      const int32_t a1 = (int32_t)(rowA0 + 127 < C - 1 ? rowA0 + 127 : C - 1);
      loA_min = p.doc_start[g0 + (int32_t)rowA0];
      loA_max = p.doc_start[g0 + a1];
      if (validB) {
        const int32_t b1 = (int32_t)(rowA0 + 255 < C - 1 ? rowA0 + 255 : C - 1);
        loB_min = p.doc_start[g0 + (int32_t)rowA0 + 128];
        loB_max = p.doc_start[g0 + b1];
      }
      // keys before loA_min (<= loB_min) are invisible to every row: only
      // chunks [loA_min / C, gq] can hold visible keys; at step s the rank
      // holds the K/V of rank (r - s) mod P
      ring.build(loA_min / (int32_t)C, gq, P, r, -1, s, se);
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
          if (s >= se) return false;
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
        kchunk0 = gk * (int32_t)C;
        if (skip) continue;
        // whole chunk before every row's document
        const int32_t klast_chunk = kchunk0 + (int32_t)C - 1;
        if (DOC && klast_chunk < loA_min && (!validB || klast_chunk < loB_min)) continue;
        int64_t last = rowA0 + (validB ? 255 : 127);
        if (last > C - 1) last = C - 1;
        tmax = diag ? (int)(last / BN) : ntiles - 1;
        // tiles wholly before every row's document hold no visible key
        t = (DOC && loA_min > kchunk0) ? (int)((loA_min - kchunk0) / BN) : 0;
        in_chunk = true;
      }
      if (t > tmax) {
        in_chunk = false;
        continue;
      }
      key0 = t * BN;
      ++t;
      kglob0 = kchunk0 + key0;
      const int32_t klast = kchunk0 + (int32_t)((int64_t)key0 + BN - 1 < C - 1 ? (int64_t)key0 + BN - 1 : C - 1);
      actA = validA && (!diag || key0 <= rowA0 + 127) && (!DOC || klast >= loA_min);
      actB = validB && (!diag || key0 <= rowA0 + 255) && (!DOC || klast >= loB_min);
      if (!(actA || actB)) continue;
      const bool tail = (int64_t)key0 + BN > C;
      maskA = (diag && (int64_t)key0 + BN - 1 > rowA0) || tail || (DOC && kglob0 < loA_max);
      maskB = (diag && (int64_t)key0 + BN - 1 > rowA0 + 128) || tail || (DOC && kglob0 < loB_max);
      kv_row = base_row + key0;
      return true;
    }
  }
};

template <int D>
struct Smem {
  static constexpr int QT = BM * D * 2;   // one Q tile
  static constexpr int KT = BN * D * 2;   // one K or V tile (a ring stage)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = 2 * QT;
  static constexpr int OFF_BAR = OFF_KV + NSTAGE * KT;
  static constexpr int NBAR = 2 * NSTAGE + 2 + 5 * 2;
  static constexpr int BYTES = OFF_BAR + NBAR * 8 + 16;
  static constexpr int ALLOC = BYTES + 1024;  // slack for 1024-byte alignment
};

template <int D, bool DOC>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ Params p) {
  using L = Smem<D>;
  constexpr int NH = D / 64;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const uint32_t sQ0 = base + L::OFF_Q, sQ1 = sQ0 + L::QT;
  const uint32_t sKV = base + L::OFF_KV;
  const uint32_t bar0 = base + L::OFF_BAR;
  auto kv_full = [&](int i) { return bar0 + 8u * i; };
  auto kv_empty = [&](int i) { return bar0 + 8u * (NSTAGE + i); };
  const uint32_t q_full = bar0 + 8u * (2 * NSTAGE);
  const uint32_t q_empty = q_full + 8u;
  auto s_full = [&](int x) { return q_empty + 8u + 8u * x; };
  auto s_free = [&](int x) { return q_empty + 24u + 8u * x; };
  auto p_full = [&](int x) { return q_empty + 40u + 8u * x; };
  auto o_done = [&](int x) { return q_empty + 56u + 8u * x; };
  auto o_free = [&](int x) { return q_empty + 72u + 8u * x; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::OFF_BAR + L::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::OFF_BAR + L::NBAR * 8 + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSTAGE; ++i) {
      mbar_init(kv_full(i), 1);
      mbar_init(kv_empty(i), 2);  // one release per MMA issuer
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 2);
    for (int x = 0; x < 2; ++x) {
      mbar_init(s_full(x), 1);
      mbar_init(s_free(x), 4);
      mbar_init(p_full(x), 4);
      mbar_init(o_done(x), 1);
      mbar_init(o_free(x), 4);
    }
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
  if (warp < 4) {
  setmaxnreg_dec<kRegCtl>();
  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    // The whole warp runs the (uniform) control flow; lane 0 issues.
    {
      const uint32_t leader = lane == 0 ? 1u : 0u;
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
      }
      int64_t pos = 0;
      uint32_t qcnt = 0;
      for (int64_t idx = blockIdx.x; idx < p.n_items; idx += gridDim.x) {
        const Item it = decode_item(p, idx);
        if (qcnt > 0) mbar_wait(q_empty, (qcnt - 1) & 1, abort_flag, cap);
        mbar_arrive_expect_tx_w(leader, q_full, (uint32_t)((it.validA ? 1 : 0) + (it.validB ? 1 : 0)) * L::QT);
        const int rowA = (int)((int64_t)it.r * 2 * p.C + (int64_t)it.c * p.C + it.rowA0);
#pragma unroll
        for (int hf = 0; hf < NH; ++hf) {
          tma_load_3d_w(leader, sQ0 + hf * HALF, &tmQ, q_full, hf * 64, it.h, rowA);
          if (it.validB) tma_load_3d_w(leader, sQ1 + hf * HALF, &tmQ, q_full, hf * 64, it.h, rowA + 128);
        }
        ++qcnt;
        TileIter<DOC> ti(p, it);
        while (ti.next()) {
#pragma unroll
          for (int kv = 0; kv < 2; ++kv) {
            const int st = (int)(pos % NSTAGE);
            const uint32_t use = (uint32_t)(pos / NSTAGE);
            mbar_wait(kv_empty(st), (use & 1) ^ 1, abort_flag, cap);
            mbar_arrive_expect_tx_w(leader, kv_full(st), L::KT);
#pragma unroll
            for (int hf = 0; hf < NH; ++hf)
              tma_load_3d_w(leader, sKV + st * L::KT + hf * HALF, kv ? (const void*)&tmV : (const void*)&tmK,
                            kv_full(st), hf * 64, it.kvh, (int)ti.kv_row);
            ++pos;
          }
        }
      }
      // Drain: every load issued must have landed before the CTA exits.
      volatile int no_abort = 0;
      for (int64_t i = (pos > NSTAGE ? pos - NSTAGE : 0); i < pos; ++i)
        mbar_wait(kv_full((int)(i % NSTAGE)), (uint32_t)((i / NSTAGE) & 1), &no_abort, cap);
      if (qcnt > 0) mbar_wait(q_full, (qcnt - 1) & 1, &no_abort, cap);
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------- MMA issuers
    // Warp 1 issues tile A's MMAs, warp 2 tile B's: S_X = Q_X K^T and
    // O_X += P_X V, each issuer in its own order (PV_X(j), then S_X(j+1),
    // which overwrites P_X(j) only after PV_X(j) has read it: one thread's
    // tcgen05 MMAs run in issue order). While one issuer waits for its P or
    // does its bookkeeping, the other's MMAs keep the tensor core busy. Each
    // K/V stage and the Q tiles are released once by each issuer: a commit if
    // it read them, a plain arrival once the stage has filled if its tile had
    // nothing to do there. The whole warp runs the (uniform) control flow and
    // computes the descriptors; lane 0 issues the tcgen05 instructions.
    //
    // Without document masks every item is a long run of K/V tiles, and two
    // free-running issuers let the softmax groups drift into phase, where
    // they contend for the exponential unit. There an issue token keeps the
    // order A, B, A, B per K/V step: named barrier 1 passes it from A to B,
    // barrier 2 from B back to A (64 threads each: both issuer warps). Items
    // of packed documents are short; there the issuers run free.
    {
      constexpr bool kOrdered = !DOC;
      const int x = warp - 1;  // 0: tile A, 1: tile B
      const uint32_t leader = lane == 0 ? 1u : 0u;
      constexpr uint32_t idS = idesc_bf16_f32(BM, BN, 0, 0);
      constexpr uint32_t idO = idesc_bf16_f32(BM, D, 0, 1);
      const uint32_t tSx = tmem + (uint32_t)(x * 128);
      const uint32_t tOx = tmem + 256u + (uint32_t)(x * D);
      // operand descriptors, computed once: this issuer's Q tile, and stage 0
      // of the K/V ring (stage s is (s * KT) >> 4 further)
      const uint64_t dQx = desc_kmajor_sw128(x ? sQ1 : sQ0);
      const uint64_t dK0 = desc_kmajor_sw128(sKV);
      const uint64_t dV0 = desc_mnmajor_sw128(sKV, HALF);
      const uint32_t bar_s_full = s_full(x), bar_s_free = s_free(x), bar_p_full = p_full(x);
      const uint32_t bar_o_done = o_done(x), bar_o_free = o_free(x);
      uint32_t pos = 0;  // K/V ring position (stage pos % NSTAGE)
      uint32_t qcnt = 0, s_cnt = 0, pv_cnt = 0, epi_cnt = 0;
      uint32_t groups = 0;  // K/V steps this issuer has passed the token for
      bool first_pv = true;

      // Both issuers walk the same items and K/V steps, so every token taken
      // is passed and every named-barrier phase completes, abort included
      // (an aborted wait returns at once and the walk goes on).
      auto take_token = [&]() {
        if constexpr (kOrdered) {
          __syncwarp();
          if (x == 0) {
            if (groups > 0) asm volatile("bar.sync 2, 64;" ::: "memory");
          } else {
            asm volatile("bar.sync 1, 64;" ::: "memory");
          }
        }
      };
      auto pass_token = [&]() {
        if constexpr (kOrdered) {
          __syncwarp();
          if (x == 0) asm volatile("bar.arrive 1, 64;" ::: "memory");
          else asm volatile("bar.arrive 2, 64;" ::: "memory");
          ++groups;
        }
      };
      auto wait_full = [&](uint32_t ps) {
        mbar_wait(kv_full((int)(ps % NSTAGE)), (ps / NSTAGE) & 1, abort_flag, cap);
      };
      auto release = [&](uint32_t ps, bool used) {  // this issuer is done with stage ps
        if (used) mma_commit_w(leader, kv_empty((int)(ps % NSTAGE)));
        else if (leader) mbar_arrive(kv_empty((int)(ps % NSTAGE)));
      };
      auto wait_s_free = [&]() {  // the softmax has read S_X (and P_X was consumed)
        if (s_cnt > 0) mbar_wait(bar_s_free, (s_cnt - 1) & 1, abort_flag, cap);
      };
      auto mma_S = [&](uint32_t kpos) {  // S_X = Q_X K^T
        const uint64_t dk = dK0 + (uint64_t)((kpos % NSTAGE) * (L::KT >> 4));
        if (leader) {
          mma_ss_kblock<D / 16, HALF>(tSx, dQx, dk, idS, 0u);
          mma_commit(bar_s_full);
        }
        ++s_cnt;
      };
      auto mma_PV = [&](uint32_t vpos) {  // O_X += P_X V
        const uint64_t dv = dV0 + (uint64_t)((vpos % NSTAGE) * (L::KT >> 4));
        // P_X is in TMEM over the first 64 columns of S_X (8 columns = 16
        // keys per instruction)
        if (leader) {
          mma_ts_kblock<BN / 16>(tOx, tSx, dv, idO, first_pv ? 0u : 1u);
          mma_commit(bar_o_done);
        }
        ++pv_cnt;
        first_pv = false;
      };

      for (int64_t idx = blockIdx.x; idx < p.n_items; idx += gridDim.x) {
        const Item it = decode_item(p, idx);
        mbar_wait(q_full, qcnt & 1, abort_flag, cap);
        ++qcnt;
        first_pv = true;
        TileIter<DOC> ti(p, it);
        bool has = ti.next();
        bool act = false;
        if (has) {
          act = x ? ti.actB : ti.actA;
          const uint32_t kpos = pos++;
          wait_full(kpos);
          if (act) wait_s_free();
          take_token();
          if (act) {
            tc_fence_after();
            mma_S(kpos);
          }
          release(kpos, act);
          pass_token();
        }
        while (has) {
          const bool cur = act;
          const uint32_t vpos = pos++;
          wait_full(vpos);
          // the next tile's bookkeeping and waits come first, so that
          // S_X(j+1) follows PV_X(j) in the tensor pipe without a gap
          const bool has_next = ti.next();
          const bool nxt = has_next && (x ? ti.actB : ti.actA);
          uint32_t kn = 0;
          if (has_next) {
            kn = pos++;
            wait_full(kn);
          }
          if (cur) {  // P_X written; O_X free at an item's first PV
            mbar_wait(bar_p_full, pv_cnt & 1, abort_flag, cap);
            if (first_pv && epi_cnt > 0) mbar_wait(bar_o_free, (epi_cnt - 1) & 1, abort_flag, cap);
          }
          if (nxt) wait_s_free();
          take_token();
          tc_fence_after();
          if (cur) mma_PV(vpos);
          release(vpos, cur);
          if (nxt) mma_S(kn);
          if (has_next) release(kn, nxt);
          pass_token();
          act = nxt;
          has = has_next;
        }
        mma_commit_w(leader, q_empty);
        if (!first_pv) ++epi_cnt;
      }
      if constexpr (kOrdered) {
        // take tile B's last token, so that barrier 2 ends with no phase open
        __syncwarp();
        if (x == 0 && groups > 0) asm volatile("bar.sync 2, 64;" ::: "memory");
      }
    }
  }
  } else {
  setmaxnreg_inc<kRegSoftmax>();
  {
    // --------------------------------------------------- softmax groups
    const int grp = (warp - 4) >> 2;  // 0: tile A, 1: tile B
    const int wq = warp & 3;           // TMEM lane quarter this warp may access
    const int row = wq * 32 + lane;    // row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + (uint32_t)(grp * 128) + lane_off;
    const uint32_t tO = tmem + 256u + (uint32_t)(grp * D) + lane_off;
    const float sl2 = p.scale_log2;
    uint32_t s_cnt = 0, pv_cnt = 0;

    for (int64_t idx = blockIdx.x; idx < p.n_items; idx += gridDim.x) {
      const Item it = decode_item(p, idx);
      const bool valid = grp ? it.validB : it.validA;
      if (!valid) continue;
      const int64_t rin = it.rowA0 + grp * 128 + row;  // row within the chunk
      // first visible key (global position) of this row's document
      const int32_t gqrow = (it.c ? 2 * p.P - 1 - it.r : it.r) * (int32_t)p.C + (int32_t)rin;
      const int32_t lo_row = (DOC && rin < p.C) ? p.doc_start[gqrow] : 0;
      // m: stored running max (log2 units); l: running sum of the fp32
      // probabilities; mxg: the row's largest raw score so far (document
      // build only, see the epilogue).
      float m = -CUDART_INF_F, l = 0.f, mxg = -CUDART_INF_F;
      int n_pv = 0;
      TileIter<DOC> ti(p, it);
      while (ti.next()) {
        if (!(grp ? ti.actB : ti.actA)) continue;
        const bool msk = grp ? ti.maskB : ti.maskA;
        mbar_wait(s_full(grp), s_cnt & 1, abort_flag, cap);
        ++s_cnt;
        tc_fence_after();
        int64_t lim = 128;  // visible columns of this row in the tile: [lb, lim)
        int32_t lb = 0;
        if (msk) {
          lim = ti.C - ti.key0;
          if (ti.diag) {
            const int64_t dl = rin - ti.key0 + 1;
            lim = dl < lim ? dl : lim;
          }
          if (DOC) lb = lo_row - ti.kglob0;
        }
        // The per-tile softmax, compiled twice: with the causal / ragged-tail
        // / document mask (diagonal, last and boundary tiles) and without it.
        // One TMEM read per tile: the thread's whole row of S (128 fp32)
        // stays in registers for the max and the exponentials.
        float alpha = 1.f, rs = 0.f;
        bool need = false;
        auto tile = [&](auto MKc) {
          constexpr bool MK = decltype(MKc)::value;
          uint32_t sr[128];
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tmem_ld32(tS + 32u * c, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
          tmem_wait_ld();
          if (MK) {  // masked columns become -inf: their exponential is 0
#pragma unroll
            for (int j = 0; j < 128; ++j)
              if (!(j < lim && j >= lb)) sr[j] = 0xff800000u;
          }
          // row max: four independent chains of three-input maxima over
          // columns 0-3 (seeds), 4-123 (15 rounds of 8) and 124-127
          float mxv[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) mxv[u] = __uint_as_float(sr[u]);
#pragma unroll
          for (int j = 4; j < 124; j += 8) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
              mxv[u] = max3f(mxv[u], __uint_as_float(sr[j + 2 * u]), __uint_as_float(sr[j + 2 * u + 1]));
          }
          mxv[0] = max3f(mxv[0], __uint_as_float(sr[124]), __uint_as_float(sr[125]));
          mxv[1] = max3f(mxv[1], __uint_as_float(sr[126]), __uint_as_float(sr[127]));
          const float mx = max3f(mxv[0], mxv[1], fmaxf(mxv[2], mxv[3]));
          const float mc = fmaxf(m, mx * sl2);
          // P is rounded to bf16 for the PV product, so the row's largest
          // probability must be exactly 1 or have its rounding error taken
          // out: otherwise that dominant term is up to 2^-9 off, which on
          // rows with few visible keys alone exceeds the output tolerance.
          // Without documents the max is raised whenever a tile holds a
          // larger score (the largest probability is then exactly 1). With
          // documents rows are short and that would rescale O at almost
          // every tile, so the max is raised only past a 2^8 margin and the
          // epilogue corrects the dominant term instead.
          if constexpr (DOC) {
            need = mc > m + 8.0f;
            mxg = fmaxf(mxg, mx);
          } else {
            need = mc > m;
          }
          alpha = 1.f;
          if (need) {
            alpha = ex2_approx(m - mc);
            m = mc;
          }
          const float mu = (m == -CUDART_INF_F) ? 0.f : m;
          // The previous PV of this group is complete (it was issued before
          // this S and tcgen05 work completes in order); the wait is cheap and
          // makes the P buffer reuse explicit.
          if (pv_cnt > 0) {
            mbar_wait(o_done(grp), (pv_cnt - 1) & 1, abort_flag, cap);
            tc_fence_after();
          }
          // P = 2^(s*scale*log2e - m) as bf16 pairs written back into TMEM
          // over the first 64 columns of S (key pair u in column u); the PV
          // MMA reads it there. Scale-and-shift and the row sums run as
          // packed fp32 pairs.
          const float2 sl2v = make_float2(sl2, sl2), nmu = make_float2(-mu, -mu);
          float2 rsv[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                           make_float2(0.f, 0.f)};
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t pk[32];
#pragma unroll
            for (int u = 0; u < 32; ++u) {
              const int j0 = 64 * hh + 2 * u;
              const float2 x =
                  fma_f32x2(make_float2(__uint_as_float(sr[j0]), __uint_as_float(sr[j0 + 1])), sl2v, nmu);
              const float2 e = make_float2(ex2_approx(x.x), ex2_approx(x.y));
              rsv[u & 3] = add_f32x2(rsv[u & 3], e);
              pk[u] = pack_bf16x2_alu(e.x, e.y);
            }
            tmem_st32(tS + 32u * hh, pk);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_free(grp));
          const float2 r01 = add_f32x2(rsv[0], rsv[1]), r23 = add_f32x2(rsv[2], rsv[3]);
          const float2 r = add_f32x2(r01, r23);
          rs = r.x + r.y;
        };
        if (msk) tile(std::true_type{});
        else tile(std::false_type{});
        l = l * alpha + rs;
        if (n_pv > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + 32u * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
            tmem_st32(tO + 32u * c, o);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(grp));
        ++pv_cnt;
        ++n_pv;
      }

      // ---------------------------------------------------------- epilogue
      // O = acc / (l + c) and LSE = (m + log2 l) ln 2, merged into the
      // running state when accumulating; written 32 columns at a time.
      // Document build: c is the bf16 rounding error of the row's largest
      // probability, added to the normaliser of O only. The stored max never
      // changes after the tile that holds the row's largest score (that tile
      // either raised it to the score, or the score is within 2^8 of it, and
      // so is every later tile's max), so that element was computed with the
      // final shift: the same fma, exponential and rounding as the tile
      // (pack_bf16x2_alu) reproduce it here. Without documents c = 0.
      const float LN2 = 0.6931471805599453f;
      float lse_new = -CUDART_INF_F;
      float inv = 0.f;
      if (l > 0.f) {
        lse_new = (m + log2f(l)) * LN2;
        float c = 0.f;
        if constexpr (DOC) {
          const float e = ex2_approx(fmaf(mxg, sl2, -m));
          c = __uint_as_float((__float_as_uint(e) + 0x8000u) & 0xFFFF0000u) - e;
        }
        inv = 1.f / (l + c);
      }
      const bool row_ok = rin < p.C;
      const int64_t lrow = (int64_t)it.r * 2 * p.C + (int64_t)it.c * p.C + rin;
      const int64_t rh = lrow * p.Hq + it.h;
      float wa = 0.f, wb = inv, L = lse_new;
      float4* oacc = (p.o_acc && row_ok) ? reinterpret_cast<float4*>(p.o_acc + rh * D) : nullptr;
      if (p.accumulate && row_ok) {
        const float lo = p.lse[rh];
        const float mm = fmaxf(lo, lse_new);
        if (mm == -CUDART_INF_F) {
          wb = 0.f;
          L = -CUDART_INF_F;
        } else {
          const float ea = expf(lo - mm), eb = expf(lse_new - mm);
          const float sum = ea + eb;
          L = mm + logf(sum);
          wa = ea / sum;
          wb = inv * (eb / sum);
        }
      }
      if (row_ok) p.lse[rh] = L;
      if (n_pv > 0) {
        mbar_wait(o_done(grp), (pv_cnt - 1) & 1, abort_flag, cap);
        tc_fence_after();
      }
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t acc[32];
        if (n_pv > 0) {
          tmem_ld32(tO + 32u * c, acc);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) acc[j] = 0u;
        }
        if (row_ok) {
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            float4 v;
            v.x = __uint_as_float(acc[j + 0]) * wb;
            v.y = __uint_as_float(acc[j + 1]) * wb;
            v.z = __uint_as_float(acc[j + 2]) * wb;
            v.w = __uint_as_float(acc[j + 3]) * wb;
            const int q4 = (32 * c + j) / 4;
            if (p.accumulate) {
              const float4 old = oacc[q4];
              v.x += wa * old.x;
              v.y += wa * old.y;
              v.z += wa * old.z;
              v.w += wa * old.w;
            }
            if (oacc) oacc[q4] = v;
            if (p.finalize) {
              uint2 bb;
              bb.x = pack_bf16x2(v.x, v.y);
              bb.y = pack_bf16x2(v.z, v.w);
              reinterpret_cast<uint2*>(p.o_out + rh * D)[q4] = bb;
            }
          }
        }
      }
      if (n_pv > 0) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_free(grp));
      }
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

}  // namespace fwd
}  // namespace mmsp
