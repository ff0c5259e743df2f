// fwd_pair_sm100.cuh -- the dense 16-bit forward (D = 128) on CTA pairs for sm_100a.
//
// Method: the online-softmax forward of the StreamAttention page ("Kernel Design (Fused
// Online Softmax)") exactly as attn_fwd_sm100 computes it -- the same unit order, masks,
// lazy reference (moved past 2^8), exponentials (one pair in four on the FMA pipe), rounded
// and unrounded row sums (kept per 64-key half and added at the end), epilogue -- so the two
// kernels give identical bits.  A different machine layout:
//
//   * a cluster of two CTAs on two SMs runs each unit (batch, head, 256 query rows): CTA r
//     owns query rows 128 r .. 128 r + 127 of it.  The products are 2-SM tensor-core
//     instructions (cta_group::2, M = 256) issued by the leader CTA (rank 0): each CTA keeps
//     its own Q rows and its half of every K tile (64 keys) and V tile (64 of the 128 value
//     columns) in shared memory, and its 128 rows of S and O in tensor memory, so a K/V
//     tile is loaded once per pair and every SM loads half of it;
//   * with one Q tile per SM, tensor memory holds S twice (columns 0-127 and 128-255) next
//     to O (256-383): the product S(j+2) = Q K_{j+2}^T is issued right behind P(j) V_j, while
//     the softmax works on S(j+1) -- the softmax never waits for its own tile's next S, so a
//     K/V step costs max(tensor time, softmax time) instead of their sum;
//   * the softmax of a CTA's 128 rows runs on 8 warps: warpgroup h (warps 4 + 4h .. 7 + 4h)
//     takes keys 64 h .. 64 h + 63 of each row; the two halves of a row exchange their
//     maxima through shared memory (a 64-thread named barrier per lane quarter), agree on
//     the reference, and write their halves of P into their own S columns (keys 0-63 over S
//     columns 0-31, keys 64-127 over columns 96-127), so neither overwrites what the other
//     still reads.  Warpgroup 0 also rescales O when the reference moves, after the previous
//     P V has completed (it waits for that completion at every step, late in the step); once
//     P is handed over, the next step's S starts loading from tensor memory;
//   * loads: each CTA's load warp brings its own Q rows and K/V halves into its own shared
//     memory, the bytes counted on the leader's barrier (pair loads, no multicast), so the
//     leader's MMA warp waits once per tile for both halves.  Commits arrive in both CTAs
//     (multicast to the pair); the softmax warps of both CTAs arrive on the leader's P
//     barrier, and the completion of a step's P V is read from its V slot's free barrier.
// Launched with clusters of two CTAs.  Static unit order only (the snake of fwd_unit_of over
// the clusters); every wait is bounded.
#pragma once
#include "fwd_sm100.cuh"

namespace sa {

struct PairCfg {
  static constexpr int D = 128;
  static constexpr int Q_BYTES = 2 * 128 * 128;      // 128 rows x 128 elements: two 16 KB boxes
  static constexpr int Q_BUFS = 2;                   // Q of the next unit loads during this one
  static constexpr int HALF_BYTES = 16384;           // a CTA's half of a K or V tile
  static constexpr int K_BOX_BYTES = 64 * 128;       // K half: 64 keys x 128 bytes per 64-element box
  static constexpr int STAGES = 8;                   // ring slots (K and V halves)
  static constexpr int SMEM_BARS = 1024;
  static constexpr int SMEM_X = 4096;                // maxima (2 steps x 2 halves x 128) + sums (2 x 2 x 128)
  static constexpr int SMEM_TOTAL = 1024 + Q_BUFS * Q_BYTES + STAGES * HALF_BYTES + SMEM_BARS + SMEM_X;
  static constexpr int THREADS = 384;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t O_COL = 256;
  __host__ __device__ static constexpr uint32_t S_COL(int b) { return 128u * b; }
  // P of keys 64 h .. 64 h + 63 (16-bit pairs, 32 columns) inside S buffer b
  __host__ __device__ static constexpr uint32_t P_COL(int b, int h) { return 128u * b + (h ? 96u : 0u); }
};

struct PairSmem {
  uint8_t* q;          // [Q_BUFS][2 boxes][128 rows][128 B]
  uint8_t* ring;       // [STAGES][16 KB]
  uint64_t* kv_full;   // [STAGES] (leader) both CTAs' halves landed
  uint64_t* kv_empty;  // [STAGES] slot read by the pair's products (multicast commit)
  uint64_t* q_full;    // [Q_BUFS] (leader) both CTAs' Q rows landed
  uint64_t* q_empty;   // [Q_BUFS] Q read by the unit's last S product (multicast commit)
  uint64_t* s_full;    // [2] S buffer written (multicast commit)
  uint64_t* p_full;    // [2] (leader) P of buffer b written in both CTAs (16 warps)
  uint64_t* o_done;    // the unit's last P V complete (multicast commit)
  uint64_t* o_free;    // (leader) both CTAs' epilogues have read O (16 warps)
  uint64_t* fin;       // every product of the pair complete (multicast commit)
  uint32_t* tmem_holder;
  volatile int* abort_flag;
  float* xmax;         // [2 step parities][2 halves][128 rows]
  float* xsum;         // [2 halves][2 sums][128 rows]
  __device__ explicit PairSmem(uint8_t* s) {
    q = s;
    ring = s + PairCfg::Q_BUFS * PairCfg::Q_BYTES;
    uint64_t* b = (uint64_t*)(ring + PairCfg::STAGES * PairCfg::HALF_BYTES);
    kv_full = b;
    kv_empty = b + PairCfg::STAGES;
    uint64_t* c = b + 2 * PairCfg::STAGES;
    q_full = c; q_empty = c + 2;
    s_full = c + 4;            // [2]
    p_full = c + 6;            // [2]
    o_done = c + 8; o_free = c + 9; fin = c + 10;
    tmem_holder = (uint32_t*)(c + 11);
    abort_flag = (volatile int*)(tmem_holder + 1);
    xmax = (float*)(ring + PairCfg::STAGES * PairCfg::HALF_BYTES + PairCfg::SMEM_BARS);
    xsum = xmax + 2 * 2 * 128;
  }
};

// The K/V ring order of a unit of n steps, shared by the load warp, the MMA warp and the
// softmax: K0, K1, then for each step j: V_j, K_{j+2}.  Item i is K or V of key tile `tile`.
__device__ __forceinline__ int pair_seq_len(int n) { return 2 * n; }
__device__ __forceinline__ void pair_seq_item(int i, int n, bool& is_k, int& tile) {
  const int head = n > 1 ? 2 : 1;                 // K0 (and K1) first
  if (i < head) { is_k = true; tile = i; return; }
  const int r = i - head;                         // then V_j, K_{j+2} alternating while j + 2 < n
  const int pairs = n > 2 ? n - 2 : 0;            // steps j with a K_{j+2} behind their V_j
  if (r < 2 * pairs) { is_k = (r & 1); tile = is_k ? r / 2 + 2 : r / 2; return; }
  is_k = false;
  tile = pairs + (r - 2 * pairs);                 // the last one or two V tiles
}
// Position of V_j in the unit's sequence.
__device__ __forceinline__ int pair_seq_pos_v(int j, int n) {
  const int head = n > 1 ? 2 : 1, pairs = n > 2 ? n - 2 : 0;
  return j < pairs ? head + 2 * j : head + 2 * pairs + (j - pairs);
}

// ------------------------------------------------------------------ loads (both CTAs)
__device__ __forceinline__ void pair_producer(const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                                              const CUtensorMap* tm_v, const FwdParams& p, const PairSmem& sm,
                                              uint32_t rank, int cl, int ncl) {
  // both CTAs count their bytes on the leader's barriers; the leader expects both halves
  const uint32_t kv_full0 = map_shared_rank(sm.kv_full, 0), q_full0 = map_shared_rank(sm.q_full, 0);
  int ring_n = 0, q_loads = 0;
  bool ok = true;
  for (int n = 0; ok; ++n) {
    const int u = fwd_unit_of(n, cl, ncl);
    if (u >= p.n_units) break;
    const UnitInfo x = fwd_unit<false>(p, u);
    const int steps = x.nkv_max;
    if (steps == 0) continue;
    // Q rows of this CTA (zeros past the sequence), into the unit's Q buffer
    const int qb = q_loads % PairCfg::Q_BUFS;
    if (q_loads >= PairCfg::Q_BUFS) {
      ok = mbar_wait(&sm.q_empty[qb], ((q_loads / PairCfg::Q_BUFS) - 1) & 1, sm.abort_flag, 31);
      if (!ok) break;
    }
    if (rank == 0) mbar_arrive_expect_tx(&sm.q_full[qb], 2 * PairCfg::Q_BYTES);
#pragma unroll
    for (int c = 0; c < 2; ++c)
      tma_load_4d_pair(sm.q + qb * PairCfg::Q_BYTES + c * 16384, tm_q, q_full0 + qb * 8, c * 64, x.h,
                       x.qbase + x.q0 + (int)rank * 128, x.mb);
    ++q_loads;
    for (int i = 0; i < pair_seq_len(steps) && ok; ++i) {
      bool is_k;
      int kt;
      pair_seq_item(i, steps, is_k, kt);
      const int slot = ring_n % PairCfg::STAGES;
      if (ring_n >= PairCfg::STAGES) {
        ok = mbar_wait(&sm.kv_empty[slot], ((ring_n / PairCfg::STAGES) - 1) & 1, sm.abort_flag, 32);
        if (!ok) break;
      }
      uint8_t* dst = sm.ring + slot * PairCfg::HALF_BYTES;
      if (rank == 0) mbar_arrive_expect_tx(&sm.kv_full[slot], 2 * PairCfg::HALF_BYTES);
      const uint32_t bar = kv_full0 + slot * 8;
      if (is_k) {
        // keys 64 r .. 64 r + 63 of the tile, both 64-element halves of the head dimension
        const int krow = x.kbase + kt * 128 + (int)rank * 64;
        tma_load_4d_pair(dst, tm_k, bar, 0, x.kvh, krow, x.mb);
        tma_load_4d_pair(dst + PairCfg::K_BOX_BYTES, tm_k, bar, 64, x.kvh, krow, x.mb);
      } else {
        // value columns 64 r .. 64 r + 63 of all 128 keys
        tma_load_4d_pair(dst, tm_v, bar, (int)rank * 64, x.kvh, x.kbase + kt * 128, x.mb);
      }
      ++ring_n;
    }
  }
}

// ------------------------------------------------------------------ MMA issuer (leader)
template <bool BF16>
__device__ __forceinline__ void pair_mma(const FwdParams& p, const PairSmem& sm, uint32_t tmem_base, int cl,
                                         int ncl) {
  constexpr uint32_t IDESC_QK = idesc_f16(BF16 ? 1 : 0, 256, 128, 0, 0);
  constexpr uint32_t IDESC_PV = idesc_f16(BF16 ? 1 : 0, 256, 128, 0, 1);
  const uint32_t sQ0 = smem_u32(sm.q), sRing = smem_u32(sm.ring);
  int ring_n = 0, q_use = 0, units_done = 0;
  int pu[2] = {0, 0};                    // P-buffer uses consumed (p_full phases)
  bool ok = true;
  auto wait_pos = [&](int pos) -> bool {
    return mbar_wait_warp(&sm.kv_full[pos % PairCfg::STAGES], (pos / PairCfg::STAGES) & 1, sm.abort_flag, 40);
  };
  // S(buf) = Q K^T, K at ring position pos (each CTA: its 64 keys, 2 boxes along D)
  auto issue_qk = [&](int buf, int pos, uint32_t sQ) {
    const uint32_t k_addr = sRing + (pos % PairCfg::STAGES) * PairCfg::HALF_BYTES;
    mma_pair_ss_x8(tmem_base + PairCfg::S_COL(buf), smem_desc_sw128(sQ, 16, 1024), smem_desc_sw128(k_addr, 16, 1024),
                   IDESC_QK, 0u, 16384 >> 4, PairCfg::K_BOX_BYTES >> 4);
    mma_commit_pair_warp(&sm.s_full[buf]);
    mma_commit_pair_warp(&sm.kv_empty[pos % PairCfg::STAGES]);
  };
  for (int n = 0; ok; ++n) {
    const int u = fwd_unit_of(n, cl, ncl);
    if (u >= p.n_units) break;
    const UnitInfo x = fwd_unit<false>(p, u);
    const int steps = x.nkv_max;
    if (steps == 0) continue;
    const int qb = q_use % PairCfg::Q_BUFS;
    ok = mbar_wait_warp(&sm.q_full[qb], (q_use / PairCfg::Q_BUFS) & 1, sm.abort_flag, 42);
    if (!ok) break;
    ++q_use;
    tc_fence_after();
    const uint32_t sQ = sQ0 + qb * PairCfg::Q_BYTES;
    int i = 0;                           // position in the unit's ring order
    // prologue: S(0) = Q K0^T, S(1) = Q K1^T
    for (int j = 0; j < (steps > 1 ? 2 : 1) && ok; ++j, ++i) {
      ok = wait_pos(ring_n + i);
      if (!ok) break;
      tc_fence_after();
      issue_qk(j, ring_n + i, sQ);
      if (j + 1 == steps) mma_commit_pair_warp(&sm.q_empty[qb]);   // the unit's last S product
    }
    for (int j = 0; j < steps && ok; ++j) {
      const int b = j & 1;
      // ---- O += P(j) V_j
      ok = wait_pos(ring_n + i);
      if (!ok) break;
      if (j == 0 && units_done > 0) {
        ok = mbar_wait_warp_cl(sm.o_free, (units_done - 1) & 1, sm.abort_flag, 44);   // O read by both epilogues
        if (!ok) break;
      }
      const uint32_t v_addr = sRing + ((ring_n + i) % PairCfg::STAGES) * PairCfg::HALF_BYTES;
      ok = mbar_wait_warp_cl(&sm.p_full[b], pu[b] & 1, sm.abort_flag, 45);
      if (!ok) break;
      tc_fence_after();
      mma_pair_ts_x8(tmem_base + PairCfg::O_COL, tmem_base + PairCfg::P_COL(b, 0), tmem_base + PairCfg::P_COL(b, 1),
                     smem_desc_sw128(v_addr, 16384, 1024), IDESC_PV, j > 0 ? 1u : 0u);
      ++pu[b];
      // (the V slot's free barrier doubles as "P V_j complete" for the softmax)
      mma_commit_pair_warp(&sm.kv_empty[(ring_n + i) % PairCfg::STAGES]);
      if (j + 1 == steps) mma_commit_pair_warp(sm.o_done);
      ++i;
      // ---- S(j+2) = Q K_{j+2}^T into the buffer P(j) V_j has just read (issue order keeps it behind)
      if (j + 2 < steps) {
        ok = wait_pos(ring_n + i);
        if (!ok) break;
        tc_fence_after();
        issue_qk(b, ring_n + i, sQ);
        if (j + 3 == steps) mma_commit_pair_warp(&sm.q_empty[qb]);   // the unit's last S product
        ++i;
      }
    }
    if (!ok) break;
    ring_n += pair_seq_len(steps);
    ++units_done;
  }
  mma_commit_pair_warp(sm.fin);
}

// ------------------------------------------------------------------ softmax + epilogue (both CTAs)
// One thread per (row, key half): warp 4 + 4h + q, lane l -> row 32 q + l, keys 64 h .. 64 h + 63.
template <bool BF16>
__device__ __forceinline__ void pair_softmax(const FwdParams& p, const PairSmem& sm, uint32_t tmem_base,
                                             uint32_t rank, int w8, int lane, int cl, int ncl) {
  const int h = w8 >> 2, qd = w8 & 3;
  const int row_in_tile = qd * 32 + lane;
  const uint32_t lane_addr = tmem_base + ((uint32_t)(qd * 32) << 16);
  const float c2 = p.c2;
  const uint32_t p_full0 = map_shared_rank(sm.p_full, 0), o_free0 = map_shared_rank(sm.o_free, 0);
  int su[2] = {0, 0};                        // S-buffer uses consumed (s_full phases)
  int ring_n = 0, o_n = 0;                   // the unit's first ring position; o_done phases consumed
  bool ok = true;
  for (int n = 0; ok; ++n) {
    const int u = fwd_unit_of(n, cl, ncl);
    if (u >= p.n_units) break;
    const UnitInfo x = fwd_unit<false>(p, u);
    const int steps = x.nkv_max;
    const int r0 = x.q0 + (int)rank * 128;     // this CTA's first row
    const int row = r0 + row_in_tile;
    int klim = x.sk;
    if (p.causal) klim = min(x.sk, row + x.sk - x.sq + 1);
    int kvis = x.sk;                           // keys every row of this CTA's tile sees
    if (p.causal) kvis = min(kvis, max(0, r0 + x.sk - x.sq + 1));
    const int mask_from = kvis / 128;
    float m_ref = -INFINITY, l_sum = 0.f, l_lse = 0.f;
    uint32_t v[2][32];
    // S(0) of the unit: wait and start loading this thread's 64 scores
    if (steps > 0) {
      ok = mbar_wait_warp(&sm.s_full[0], su[0] & 1, sm.abort_flag, 50);
      if (!ok) break;
      ++su[0];
      tc_fence_after();
      tmem_ld32(lane_addr + PairCfg::S_COL(0) + h * 64, v[0]);
      tmem_ld32(lane_addr + PairCfg::S_COL(0) + h * 64 + 32, v[1]);
    }
    for (int j = 0; j < steps; ++j) {
      const int b = j & 1;
      tmem_wait_ld_regs(v[0]);
      tmem_wait_ld_regs(v[1]);
      const bool full = j < mask_from && c2 >= 0.f;
      float mx[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
      if (full) {
        chunk_max(v[0], mx);
        chunk_max(v[1], mx);
      } else {
        const int kl = klim - j * 128 - h * 64;   // my keys >= kl are invisible
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int t = 0; t < 32; ++t)
            v[c][t] = __float_as_uint((c * 32 + t < kl) ? __uint_as_float(v[c][t]) * c2 : -INFINITY);
          chunk_max(v[c], mx);
        }
      }
      float mine = max_of8(mx);
      if (full) mine *= c2;
      // the two halves of the row agree on the tile max
      float* xm = sm.xmax + b * 256;
      xm[h * 128 + row_in_tile] = mine;
      asm volatile("bar.sync %0, 64;" ::"r"(2 + qd) : "memory");
      const float m_tile = fmaxf(mine, xm[(1 - h) * 128 + row_in_tile]);
      const bool need = m_tile > m_ref + kRescaleThresh;
      float alpha = 1.f;
      if (need) {
        alpha = ex2(m_ref - m_tile);             // 0 when m_ref == -inf
        l_sum *= alpha;
        l_lse *= alpha;
        m_ref = m_tile;
      }
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      const f32x2 scale2 = full ? pack_f2(c2, c2) : pack_f2(1.f, 1.f), negm2 = pack_f2(-m_use, -m_use);
      f32x2 rse2[2] = {0ull, 0ull};
      float rs[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t pa = lane_addr + PairCfg::P_COL(b, h);
      if (full) {
        softmax_chunk_any<BF16, false, kPolyEvery>(v[0], scale2, negm2, rs, rse2, pa, 0);
        softmax_chunk_any<BF16, false, kPolyEvery>(v[1], scale2, negm2, rs, rse2, pa, 1);
      } else {
        softmax_chunk_any<BF16, false, 0>(v[0], scale2, negm2, rs, rse2, pa, 0);
        softmax_chunk_any<BF16, false, 0>(v[1], scale2, negm2, rs, rse2, pa, 1);
      }
      sum_rounded(rs, l_sum);
      sum_f2x2(rse2, l_lse);
      if (h == 0 && j > 0) {
        // O holds P V up to step j-1 once that product completes (its V slot's free barrier);
        // rescale it (all 128 columns) if the reference moved.  Waited at every step.
        const int pos = ring_n + pair_seq_pos_v(j - 1, steps);
        ok = mbar_wait_warp(&sm.kv_empty[pos % PairCfg::STAGES], (pos / PairCfg::STAGES) & 1, sm.abort_flag, 52);
        if (!ok) break;
        if (__any_sync(0xffffffffu, need)) {
          tc_fence_after();
          rescale_o_row<128>(lane_addr + PairCfg::O_COL, alpha);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(p_full0 + b * 8);
      // then S(j+1) (issued before P(j) V_j, so usually complete): start loading it
      if (j + 1 < steps) {
        const int nb = (j + 1) & 1;
        ok = mbar_wait_warp(&sm.s_full[nb], su[nb] & 1, sm.abort_flag, 50 + nb);
        if (!ok) break;
        ++su[nb];
        tc_fence_after();
        tmem_ld32(lane_addr + PairCfg::S_COL(nb) + h * 64, v[0]);
        tmem_ld32(lane_addr + PairCfg::S_COL(nb) + h * 64 + 32, v[1]);
      }
    }
    if (!ok) break;
    ring_n += pair_seq_len(steps);
    // ---------------- epilogue: O / l, LSE (both halves of the row: value columns 64 h ..)
    if (steps > 0) {
      ok = mbar_wait_warp(sm.o_done, o_n & 1, sm.abort_flag, 54);
      if (!ok) break;
      ++o_n;
      tc_fence_after();
    }
    sm.xsum[(h * 2 + 0) * 128 + row_in_tile] = l_sum;
    sm.xsum[(h * 2 + 1) * 128 + row_in_tile] = l_lse;
    asm volatile("bar.sync %0, 64;" ::"r"(2 + qd) : "memory");
    // half 0's sum first: the one-CTA kernel adds its two half sums in the same order
    const float L = sm.xsum[0 * 128 + row_in_tile] + sm.xsum[2 * 128 + row_in_tile];
    const float E = sm.xsum[1 * 128 + row_in_tile] + sm.xsum[3 * 128 + row_in_tile];
    const bool store = row < x.sq;
    const float inv_l = L > 0.f ? 1.f / L : 0.f;
    using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
    T* orow = reinterpret_cast<T*>(p.o) + (((size_t)x.mb * p.Sq + x.qbase + row) * p.Hq + x.h) * 128 + h * 64;
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      uint32_t r[32];
      if (steps > 0) {
        tmem_ld32(lane_addr + PairCfg::O_COL + h * 64 + c * 32, r);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int t = 0; t < 32; ++t) r[t] = 0u;
      }
      uint32_t pk[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        const float a = __uint_as_float(r[2 * t]) * inv_l, b2 = __uint_as_float(r[2 * t + 1]) * inv_l;
        if (BF16) {
          __nv_bfloat162 h2 = __floats2bfloat162_rn(a, b2);
          pk[t] = *reinterpret_cast<uint32_t*>(&h2);
        } else {
          __half2 h2 = __floats2half2_rn(a, b2);
          pk[t] = *reinterpret_cast<uint32_t*>(&h2);
        }
      }
      if (store) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int t = 0; t < 4; ++t) dst[t] = make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
      }
    }
    if (store && h == 0 && p.lse) {
      const float lse = E > 0.f ? (m_ref + __log2f(E)) * 0.69314718055994531f : -INFINITY;
      p.lse[((size_t)x.mb * p.Hq + x.h) * p.Sq + x.qbase + row] = lse;
    }
    if (steps > 0) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(o_free0);
    }
  }
}

template <bool BF16>
__global__ void __launch_bounds__(384, 1)
attn_fwd_pair_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const PairSmem sm(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int cl = (int)cluster_id_x(), ncl = (int)nclusters_x();
  if (threadIdx.x == 0) {
    for (int i = 0; i < PairCfg::STAGES; ++i) { mbar_init(&sm.kv_full[i], 1); mbar_init(&sm.kv_empty[i], 1); }
    for (int i = 0; i < PairCfg::Q_BUFS; ++i) { mbar_init(&sm.q_full[i], 1); mbar_init(&sm.q_empty[i], 1); }
    mbar_init(&sm.s_full[0], 1); mbar_init(&sm.s_full[1], 1);
    mbar_init(&sm.p_full[0], 16); mbar_init(&sm.p_full[1], 16);
    mbar_init(sm.o_done, 1); mbar_init(sm.o_free, 16); mbar_init(sm.fin, 1);
    *sm.abort_flag = 0;
    fence_barrier_init();
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kWarpMma) {
    tmem_alloc_pair(sm.tmem_holder, PairCfg::TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == kWarpLoad && lane == 0) {
    tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  // both CTAs' barriers are initialised (and tensor memory allocated) before any arrival
  // or load completion from the other CTA
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *sm.tmem_holder;
  if (warp < 4) {
    if (warp == kWarpLoad && lane == 0) pair_producer(&tm_q, &tm_k, &tm_v, p, sm, rank, cl, ncl);
    else if (warp == kWarpMma && rank == 0) pair_mma<BF16>(p, sm, tmem_base, cl, ncl);
    __syncwarp();
  } else {
    pair_softmax<BF16>(p, sm, tmem_base, rank, warp - 4, lane, cl, ncl);
  }
  if (warp == kWarpMma) {
    // every product of the pair has completed (the leader's final commit reaches both CTAs)
    mbar_wait_warp_cl(sm.fin, 0, nullptr, 55);
  }
  if (threadIdx.x == 32 && *sm.abort_flag) {
    // a wait was abandoned: loads this CTA issued may still be in flight into its shared
    // memory (their completions count on the leader's barriers, which it cannot wait on);
    // a load lands within microseconds, so wait 100 us before the memory can go away
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 100000ull) {
    }
  }
  tc_fence_before();
  cluster_sync_all();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, PairCfg::TMEM_COLS);
  }
}

}  // namespace sa
