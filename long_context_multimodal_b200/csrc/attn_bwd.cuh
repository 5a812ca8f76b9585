// attn_bwd.cuh -- gradients of the ring-blockwise causal attention on
// tcgen05 tensor cores, all virtual ranks in one persistent launch.
//
// The pages give only the backward of the all-to-all transpose ("LongVILA
// Guide", section "Implementation", UlyssesAllToAll.backward); the gradient
// of the attention itself is a reading: with P_ij = exp(s_ij - LSE_i)
// recomputed from the saved fp32 LSE and D_i = sum_d dO_i O_i,
//   dV_j = sum_i P_ij dO_i,  dS_ij = P_ij (dO_i . v_j - D_i),
//   dQ_i = scale sum_j dS_ij k_j,  dK_j = scale sum_i dS_ij q_i,
// dK, dV summed over the query heads of each kv head.
//
// Work unit: one kv head and one tile of 128 keys of one zigzag chunk. The
// CTA keeps K and V of the tile in shared memory and dK, dV in TMEM, and
// visits every (query tile of 128 rows, query head of the group) that sees
// the keys, in ring order from the keys' point of view: at ring step s the
// block of rank k sits on rank (k + s) mod P (it was sent to the next ring
// rank s times). Per visit, five tcgen05 GEMMs (bf16 in, fp32 accumulate):
//   S^T  = K Q^T          (128 keys x 128 queries)   -> TMEM region SP
//   dP^T = V dO^T                                     -> TMEM region SP
//   dV  += P^T dO         (A = P^T from smem)         -> TMEM dV
//   dK  += dS^T Q         (A = dS^T from smem)        -> TMEM dK
//   dQ   = dS K           (A = dS^T read MN-major)    -> TMEM dQ
// dQ is read by four warps (one TMEM lane = one query row) and added into
// a fp32 dQ accumulator with 16-byte vector reductions (red.add.v4.f32);
// dK, dV are written once per unit. Units are ordered by decreasing work (keys of chunk 0
// first).
//
// Warp roles (320 threads): warp 0 TMA producer, warp 1 MMA issuer, warps
// 2-5 softmax/gradient (one thread per key = TMEM lane), warps 6-9 dQ
// readout. TMEM: SP [0,128) dV [128,256) dK [256,384) dQ [384,512).
// Shared memory: K, V (32 KB each), two Q stages, one dO stage, P^T and
// dS^T (32 KB each), two 1 KB stages of LSE*log2(e) and D.
#pragma once

#include <cuda.h>
#include <math_constants.h>

#include <type_traits>

#include "ptx.cuh"

namespace mmsp {
namespace bwd {

constexpr int BM = 128;  // keys per unit
constexpr int BN = 128;  // queries per visit
constexpr int kThreads = 320;
constexpr int HALF = 128 * 128;

struct Params {
  int32_t P, Hq, Hkv, G;
  int64_t C;        // chunk length
  int64_t Cp;       // chunk length padded to a multiple of 128 (LSE2/D rows)
  int32_t ntiles;   // 128-row tiles per chunk
  int32_t causal;
  int64_t n_units;
  float scale_log2;
  float scale;
  const float* lse2t;  // [Hq][P][2][Cp]: LSE * log2(e); +inf on padding
  const float* dt;     // [Hq][P][2][Cp]: D; 0 on padding
  float* dq_acc;       // [N][Hq][d] fp32, zeroed before the launch
  __nv_bfloat16* dk;   // [N][Hkv][d]
  __nv_bfloat16* dv;   // [N][Hkv][d]
  long long wait_cap;
};

struct Unit {
  int k, ck, kt, kvh;
  int64_t key0;  // first key of the tile within its chunk
  int gk;        // global chunk index of the keys
};

__device__ __forceinline__ Unit decode_unit(const Params& p, int64_t idx) {
  // groups of decreasing work: global key chunk 0 first
  const int64_t per_chunk = (int64_t)p.ntiles * p.Hkv;
  const int gk = (int)(idx / per_chunk);
  const int64_t w = idx - (int64_t)gk * per_chunk;
  Unit u;
  u.gk = gk;
  if (gk < p.P) {
    u.k = gk;
    u.ck = 0;
  } else {
    u.k = 2 * p.P - 1 - gk;
    u.ck = 1;
  }
  u.kvh = (int)(w / p.ntiles);
  u.kt = (int)(w % p.ntiles);
  u.key0 = (int64_t)u.kt * BM;
  return u;
}

// Enumerates the (query tile, head) visits of a unit in ring order.
struct VisitIter {
  int k, P, gk, causal, G, kvh, s, qc, t, tmax, hg, ntiles;
  int64_t C, key0, qrow_base;
  bool in_chunk;
  // current visit
  int h, r, qcur;  // query head, rank, query chunk (0/1)
  int64_t q0;      // first query row of the tile within its chunk
  int64_t lrow0;   // first rank-local row of the tile
  bool diag;

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
        if (t <= tmax) {
          q0 = (int64_t)t * BN;
          lrow0 = qrow_base + q0;
          continue;
        }
        in_chunk = false;
      }
      if (s >= P) return false;
      r = (k + s) % P;
      qcur = qc;
      const int gq = qc ? 2 * P - 1 - r : r;
      if (++qc == 2) {
        qc = 0;
        ++s;
      }
      if (causal && gq < gk) continue;
      diag = causal && gq == gk;
      // diagonal: only query tiles that reach the tile's first key
      int t0 = diag ? (int)(key0 / BN) : 0;
      tmax = ntiles - 1;
      t = t0;
      hg = 0;
      qrow_base = (int64_t)r * 2 * C + (int64_t)qcur * C;
      q0 = (int64_t)t * BN;
      lrow0 = qrow_base + q0;
      in_chunk = true;
    }
  }
};

struct Smem {
  static constexpr int TILE = 128 * 128 * 2;  // 32 KB bf16 tile (d = 128)
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = TILE;
  static constexpr int OFF_Q = 2 * TILE;        // two stages
  static constexpr int OFF_DO = 4 * TILE;       // one stage
  static constexpr int OFF_PT = 5 * TILE;
  static constexpr int OFF_DST = 6 * TILE;
  static constexpr int OFF_VEC = 7 * TILE;      // two stages x (LSE2[128], D[128])
  static constexpr int OFF_BAR = OFF_VEC + 2 * 1024;
  static constexpr int NBAR = 16;
  static constexpr int BYTES = OFF_BAR + NBAR * 8 + 16;
  // No alignment slack fits next to seven 32 KB tiles: the kernel requires a
  // 1024-byte aligned dynamic shared memory base (it is, when the kernel has
  // no static shared memory) and reports a layout error otherwise.
  static constexpr int ALLOC = BYTES;
};

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

__device__ __forceinline__ void red_add_v4_f32(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ Params p) {
  using L = Smem;
  constexpr int D = 128;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  if (base & 1023u) {
    if (threadIdx.x == 0) atomicExch(&g_timeout_flag, 2);
    return;
  }
  uint8_t* gbase = smem_raw;
  const uint32_t sK = base + L::OFF_K, sV = base + L::OFF_V;
  const uint32_t sQ0 = base + L::OFF_Q;
  const uint32_t sDO = base + L::OFF_DO;
  const uint32_t sPT = base + L::OFF_PT, sDST = base + L::OFF_DST;
  const uint32_t sVEC = base + L::OFF_VEC;
  const float* vec_g = reinterpret_cast<const float*>(gbase + L::OFF_VEC);
  const uint32_t bar0 = base + L::OFF_BAR;
  const uint32_t kv_full = bar0, kv_empty = bar0 + 8;
  auto q_full = [&](int i) { return bar0 + 16u + 8u * i; };
  auto q_empty = [&](int i) { return bar0 + 32u + 8u * i; };
  const uint32_t do_full = bar0 + 48, do_empty = bar0 + 56;
  const uint32_t sp_full = bar0 + 64, sp_free = bar0 + 72;
  const uint32_t p_full = bar0 + 80, mm_done = bar0 + 88;
  const uint32_t dq_full = bar0 + 96, dq_free = bar0 + 104;
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
    }
    mbar_init(do_full, 1);
    mbar_init(do_empty, 1);
    mbar_init(sp_full, 1);
    mbar_init(sp_free, 4);
    mbar_init(p_full, 4);
    mbar_init(mm_done, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 4);
    mbar_init(acc_full, 1);
    mbar_init(acc_free, 4);
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

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      uint32_t ucnt = 0, vis = 0;
      for (int64_t idx = blockIdx.x; idx < p.n_units; idx += gridDim.x) {
        const Unit u = decode_unit(p, idx);
        if (ucnt > 0) mbar_wait(kv_empty, (ucnt - 1) & 1, abort_flag, cap);
        mbar_arrive_expect_tx(kv_full, 2 * L::TILE);
        const int krow = (int)((int64_t)u.k * 2 * p.C + (int64_t)u.ck * p.C + u.key0);
        for (int hf = 0; hf < 2; ++hf) {
          tma_load_3d(sK + hf * HALF, &tmK, kv_full, hf * 64, u.kvh, krow);
          tma_load_3d(sV + hf * HALF, &tmV, kv_full, hf * 64, u.kvh, krow);
        }
        ++ucnt;
        VisitIter it(p, u);
        while (it.next()) {
          const int st = vis & 1;
          const uint32_t use = vis >> 1;
          mbar_wait(q_empty(st), (use & 1) ^ 1, abort_flag, cap);
          mbar_arrive_expect_tx(q_full(st), L::TILE + 1024);
          for (int hf = 0; hf < 2; ++hf)
            tma_load_3d(sQ0 + st * L::TILE + hf * HALF, &tmQ, q_full(st), hf * 64, it.h, (int)it.lrow0);
          const int64_t vrow = (((int64_t)it.h * p.P + it.r) * 2 + it.qcur) * p.Cp + it.q0;
          bulk_load(sVEC + st * 1024, p.lse2t + vrow, 512, q_full(st));
          bulk_load(sVEC + st * 1024 + 512, p.dt + vrow, 512, q_full(st));
          mbar_wait(do_empty, (vis & 1) ^ 1, abort_flag, cap);
          mbar_arrive_expect_tx(do_full, L::TILE);
          for (int hf = 0; hf < 2; ++hf) tma_load_3d(sDO + hf * HALF, &tmDO, do_full, hf * 64, it.h, (int)it.lrow0);
          ++vis;
        }
      }
      volatile int no_abort = 0;
      if (ucnt > 0) mbar_wait(kv_full, (ucnt - 1) & 1, &no_abort, cap);
      if (vis > 0) {
        mbar_wait(do_full, (vis - 1) & 1, &no_abort, cap);
        const uint32_t last = vis - 1;
        mbar_wait(q_full(last & 1), (last >> 1) & 1, &no_abort, cap);
        if (vis > 1) mbar_wait(q_full((last - 1) & 1), ((last - 1) >> 1) & 1, &no_abort, cap);
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idKQ = idesc_bf16_f32(BM, BN, 0, 0);   // S^T, dP^T
      constexpr uint32_t idGrad = idesc_bf16_f32(BM, D, 0, 1);  // dV, dK: B MN-major
      constexpr uint32_t idDQ = idesc_bf16_f32(BN, D, 1, 1);    // dQ: A and B MN-major
      const uint32_t tSP = tmem, tDV = tmem + 128u, tDK = tmem + 256u, tDQ = tmem + 384u;
      uint32_t ucnt = 0, vis = 0, spf = 0, pc = 0, dqc = 0, epi = 0;
      auto issue_kq = [&](uint32_t a, uint32_t b) {  // tSP = a[128 x d] * b[128 x d]^T
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * HALF + (kk & 3) * 32;
          mma_bf16_ss(tSP, desc_kmajor_sw128(a + off), desc_kmajor_sw128(b + off), idKQ, kk > 0 ? 1u : 0u);
        }
      };
      for (int64_t idx = blockIdx.x; idx < p.n_units; idx += gridDim.x) {
        const Unit u = decode_unit(p, idx);
        mbar_wait(kv_full, ucnt & 1, abort_flag, cap);
        ++ucnt;
        tc_fence_after();
        VisitIter it(p, u);
        bool has = it.next();
        bool first = true;
        if (has) {
          // S^T_0: the SP region is free once the previous visit's dP^T was read
          if (pc > 0) {
            mbar_wait(p_full, (pc - 1) & 1, abort_flag, cap);
            tc_fence_after();
          }
          const int st = vis & 1;
          mbar_wait(q_full(st), (vis >> 1) & 1, abort_flag, cap);
          tc_fence_after();
          issue_kq(sK, sQ0 + st * L::TILE);
          mma_commit(sp_full);
        }
        while (has) {
          const int st = vis & 1;
          // dP^T_i once S^T_i has been read
          mbar_wait(sp_free, spf & 1, abort_flag, cap);
          ++spf;
          tc_fence_after();
          mbar_wait(do_full, vis & 1, abort_flag, cap);
          tc_fence_after();
          issue_kq(sV, sDO);
          mma_commit(sp_full);
          // P^T_i, dS^T_i in shared memory (and the SP region read)
          mbar_wait(p_full, pc & 1, abort_flag, cap);
          ++pc;
          tc_fence_after();
          const bool has_next = it.next();
          if (has_next) {
            const int stn = (vis + 1) & 1;
            mbar_wait(q_full(stn), ((vis + 1) >> 1) & 1, abort_flag, cap);
            tc_fence_after();
            issue_kq(sK, sQ0 + stn * L::TILE);
            mma_commit(sp_full);
          }
          if (first && epi > 0) {
            mbar_wait(acc_free, (epi - 1) & 1, abort_flag, cap);
            tc_fence_after();
          }
          // dV += P^T dO ; dK += dS^T Q   (B operands MN-major: rows = queries)
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint32_t aoff = (kk >> 2) * HALF + (kk & 3) * 32;
            mma_bf16_ss(tDV, desc_kmajor_sw128(sPT + aoff), desc_mnmajor_sw128(sDO + kk * 2048, HALF), idGrad,
                        (kk > 0 || !first) ? 1u : 0u);
          }
          mma_commit(do_empty);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint32_t aoff = (kk >> 2) * HALF + (kk & 3) * 32;
            mma_bf16_ss(tDK, desc_kmajor_sw128(sDST + aoff),
                        desc_mnmajor_sw128(sQ0 + st * L::TILE + kk * 2048, HALF), idGrad,
                        (kk > 0 || !first) ? 1u : 0u);
          }
          mma_commit(q_empty(st));
          // dQ = dS K: A = dS^T tile read MN-major (queries contiguous, rows =
          // keys), B = K tile read MN-major (d contiguous, rows = keys)
          if (dqc > 0) {
            mbar_wait(dq_free, (dqc - 1) & 1, abort_flag, cap);
            tc_fence_after();
          }
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk)
            mma_bf16_ss(tDQ, desc_mnmajor_sw128(sDST + kk * 2048, HALF), desc_mnmajor_sw128(sK + kk * 2048, HALF),
                        idDQ, kk > 0 ? 1u : 0u);
          mma_commit(dq_full);
          mma_commit(mm_done);
          ++dqc;
          ++vis;
          first = false;
          has = has_next;
        }
        mma_commit(kv_empty);
        mma_commit(acc_full);
        ++epi;
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------- softmax / gradient rows
    const int wq = warp & 3;
    const int row = wq * 32 + lane;  // key within the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tSP = tmem + lane_off;
    const float sl2 = p.scale_log2;
    uint32_t vis = 0, spc = 0, mmc = 0, accc = 0;
    for (int64_t idx = blockIdx.x; idx < p.n_units; idx += gridDim.x) {
      const Unit u = decode_unit(p, idx);
      const int64_t kin = u.key0 + row;  // key index within its chunk
      const bool key_ok = kin < p.C;
      VisitIter it(p, u);
      while (it.next()) {
        const int st = vis & 1;
        const float* lse2 = vec_g + st * 256;
        const float* dvec = lse2 + 128;
        // visible query columns: c >= cmin (diagonal), all for key_ok
        int cmin = 0;
        if (!key_ok) cmin = 128;
        else if (it.diag) {
          const int64_t dmin = kin - it.q0;
          cmin = dmin <= 0 ? 0 : (dmin >= 128 ? 128 : (int)dmin);
        }
        // LSE2/D of this visit arrive with Q in stage st
        mbar_wait(q_full(st), (vis >> 1) & 1, abort_flag, cap);
        // S^T_i
        mbar_wait(sp_full, spc & 1, abort_flag, cap);
        ++spc;
        tc_fence_after();
        uint32_t pk[64];  // P^T row as packed bf16 pairs
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          uint32_t sr[32];
          tmem_ld32(tSP + 32u * h, sr);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const int c = 32 * h + j;
            float e0 = ex2_approx(fmaf(__uint_as_float(sr[j]), sl2, -lse2[c]));
            float e1 = ex2_approx(fmaf(__uint_as_float(sr[j + 1]), sl2, -lse2[c + 1]));
            if (c < cmin) e0 = 0.f;
            if (c + 1 < cmin) e1 = 0.f;
            pk[c / 2] = pack_bf16x2(e0, e1);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sp_free);
        // P^T / dS^T buffers free once the previous visit's MMAs completed
        if (mmc < vis) {
          mbar_wait(mm_done, mmc & 1, abort_flag, cap);
          ++mmc;
        }
#pragma unroll
        for (int c8 = 0; c8 < 16; ++c8) {
          const uint32_t addr = sPT + (c8 >> 3) * HALF + row * 128 + ((((uint32_t)c8 & 7u) ^ ((uint32_t)row & 7u)) << 4);
          st_shared_v4(addr, pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2], pk[4 * c8 + 3]);
        }
        // dP^T_i -> dS^T = P^T (dP^T - D)
        mbar_wait(sp_full, spc & 1, abort_flag, cap);
        ++spc;
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          uint32_t sr[32];
          tmem_ld32(tSP + 32u * h, sr);
          tmem_wait_ld();
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            const int c16 = 4 * h + c8;
            const uint32_t off = (c16 >> 3) * HALF + row * 128 + ((((uint32_t)c16 & 7u) ^ ((uint32_t)row & 7u)) << 4);
            uint32_t pv[4];  // this thread's own P^T values, read back from shared memory
            ld_shared_v4(sPT + off, pv);
            uint32_t o[4];
#pragma unroll
            for (int u2 = 0; u2 < 4; ++u2) {
              const int j = 8 * c8 + 2 * u2;
              const int c = 32 * h + j;
              const __nv_bfloat162 pp = *reinterpret_cast<const __nv_bfloat162*>(&pv[u2]);
              const float p0 = __low2float(pp), p1 = __high2float(pp);
              const float d0 = p0 * (__uint_as_float(sr[j]) - dvec[c]);
              const float d1 = p1 * (__uint_as_float(sr[j + 1]) - dvec[c + 1]);
              o[u2] = pack_bf16x2(d0, d1);
            }
            st_shared_v4(sDST + off, o[0], o[1], o[2], o[3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        ++vis;
      }
      // unit epilogue: dV, dK rows of this tile (dK scaled)
      mbar_wait(acc_full, accc & 1, abort_flag, cap);
      ++accc;
      tc_fence_after();
      const int64_t krow = (int64_t)u.k * 2 * p.C + (int64_t)u.ck * p.C + kin;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const uint32_t tA = tmem + 128u + 128u * which + lane_off;
        __nv_bfloat16* out = which ? p.dk : p.dv;
        const float f = which ? p.scale : 1.f;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t a[32];
          tmem_ld32(tA + 32u * c, a);
          tmem_wait_ld();
          if (key_ok) {
            uint4* dst = reinterpret_cast<uint4*>(out + (krow * p.Hkv + u.kvh) * D + 32 * c);
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
    // drain the last MMA completion so TMEM is idle before dealloc
    volatile int no_abort = 0;
    if (mmc < vis) mbar_wait(mm_done, (vis - 1) & 1, &no_abort, cap);
  } else {
    // ------------------------------------------------------ dQ readout
    const int wq = warp & 3;
    const int row = wq * 32 + lane;  // query row of the tile = TMEM lane of dQ
    const uint32_t tDQ = tmem + 384u + ((uint32_t)(wq * 32) << 16);
    const float sc = p.scale;
    uint32_t dqc = 0;
    for (int64_t idx = blockIdx.x; idx < p.n_units; idx += gridDim.x) {
      const Unit u = decode_unit(p, idx);
      VisitIter it(p, u);
      while (it.next()) {
        mbar_wait(dq_full, dqc & 1, abort_flag, cap);
        ++dqc;
        tc_fence_after();
        const bool row_ok = it.q0 + row < p.C;  // query inside the chunk
        float* dst = p.dq_acc + ((it.lrow0 + row) * p.Hq + it.h) * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t a[32];
          tmem_ld32(tDQ + 32u * c, a);
          tmem_wait_ld();
          if (c == D / 32 - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dq_free);
          }
          if (row_ok) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              red_add_v4_f32(dst + 32 * c + j, __uint_as_float(a[j]) * sc, __uint_as_float(a[j + 1]) * sc,
                             __uint_as_float(a[j + 2]) * sc, __uint_as_float(a[j + 3]) * sc);
          }
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

// D_i = sum_d dO_i * O_i (fp32) and LSE_i * log2(e), written per head into
// the padded [Hq][P][2][Cp] layout (+inf / 0 on padding rows); also zeroes
// the fp32 dQ accumulator. One warp per (local row, head); 8-byte loads.
__global__ void __launch_bounds__(256) bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                      const __nv_bfloat16* __restrict__ dout,
                                                      const float* __restrict__ lse, float* __restrict__ lse2t,
                                                      float* __restrict__ dt, float* __restrict__ dq_acc, int32_t P,
                                                      int32_t Hq, int64_t C, int64_t Cp, int zero_dq) {
  constexpr int D = 128;
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t total = (int64_t)P * 2 * Cp * Hq;  // padded (row, head) pairs
  for (int64_t w = warp; w < total; w += nwarps) {
    const int h = (int)(w % Hq);
    const int64_t pr = w / Hq;              // padded row: (r*2 + c)*Cp + t
    const int64_t t = pr % Cp;
    const int64_t rc = pr / Cp;             // r*2 + c
    const int64_t out_idx = ((int64_t)h * P * 2 + rc) * Cp + t;
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
    if (zero_dq) reinterpret_cast<float4*>(dq_acc + rh * D)[lane] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lane == 0) {
      lse2t[out_idx] = lse[rh] * 1.4426950408889634f;
      dt[out_idx] = s;
    }
  }
}

// dq (bf16, RNE) from the fp32 accumulator; 16-byte loads, 8-byte stores.
__global__ void __launch_bounds__(256) bwd_dq_convert_kernel(const float4* __restrict__ acc, uint2* __restrict__ dq,
                                                             int64_t n4) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
    const float4 v = acc[i];
    dq[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
}

}  // namespace bwd
}  // namespace mmsp
