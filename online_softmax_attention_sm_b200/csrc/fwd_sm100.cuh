// fwd_sm100.cuh -- persistent fused attention forward for sm_100a.
//
// Method: the online-softmax forward of the StreamAttention page ("Kernel Design (Fused
// Online Softmax)"): stream K/V tiles, keep per query row a running max, a running
// denominator and a rescaled accumulator, finish with acc / den and
// lse = max + log(den).  Fully masked rows follow the flash-attn-volta page's guard
// (section "Stability"): exponentiate against 0 while the running max is still -inf.
//
// B200 design:
//   * unit of work = (batch, query head, 256 query rows) = two 128-row Q tiles that
//     share every K/V tile; a persistent grid of one CTA per SM takes the units in
//     longest-first order (causal units with more K/V tiles first), each CTA fetching its
//     next unit from a global counter when it is ready for one;
//   * warp 1 (one lane) issues TMA tensor loads: the two Q tiles once per unit, then
//     K and V tiles into a ring of shared-memory slots (full/empty mbarriers);
//   * warp 0 issues tcgen05.mma (warp-uniform code, one elected lane per instruction):
//     S_t = Q_t K^T (128x128, fp32 in tensor memory) and O_t += P_t V (P_t read from
//     tensor memory, O_t fp32 in tensor memory), in the order PV_0(j), QK_0(j+1), PV_1(j),
//     QK_1(j+1) so that each softmax warpgroup works while the tensor core serves the
//     other Q tile;
//   * warpgroups 1 and 2 run the softmax of Q tile 0 and 1: each thread owns one row of
//     S (tcgen05.ld 32x32b), computes the row max, p = 2^(c*s - m) with c = scale*log2(e),
//     the row sums, writes P as 16-bit into tensor memory over S, and rescales its O row
//     only when the reference max moves by more than kRescaleThresh (exact after the
//     final division; keeps p <= 2^kRescaleThresh; FP8: past three quarters of a unit, against an
//     offset of 2^8);
//   * the epilogue (same warpgroups) divides O by the row sum, rounds to the I/O dtype
//     and writes O and the natural-log LSE.
// Causal: K/V tiles past the diagonal are never loaded or multiplied; only tiles that
// cross the diagonal or the ragged end of K are masked.
#pragma once
#include "ptx.cuh"
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <type_traits>

namespace sa {

constexpr int kUnitQueue = 4;    // unit indices the load warp may hand out ahead

// Block-sparse forward: each unit's K/V tile list, one record per (batch, head, 256-row query
// block), built by sparse_unit_lists from the caller's block mask.  A record is uint16:
// [0] list length, [1] / [2] tiles of Q tile 0 / 1, [3..7] zero, then the list (order: see
// sparse_unit_lists), each entry key tile | (Q tile 0 uses it) << 14 | (Q tile 1 uses it) << 15.
// The load warp copies a unit's record into one of kUnitQueue shared-memory slots.
constexpr int kSparseMaxKTiles = 1024;                       // keys <= 131072
constexpr int kSparseSlotBytes = 16 + 2 * kSparseMaxKTiles;  // header + longest list

// FP8: Q, K, V in e4m3 (one byte per element), the instance's products kind::f8f6f4.
template <int D, bool FP8 = false>
struct FwdCfg {
  static constexpr int BM = 128;                     // query rows per Q tile
  static constexpr int BN = 128;                     // keys per K/V tile
  static constexpr int CHUNK_ELEMS = FP8 ? 128 : 64; // elements in a 128-byte row
  static constexpr int KCH = D / CHUNK_ELEMS;        // 128-byte chunks along D
  static constexpr int CHUNK_BYTES = 128 * 128;      // one 128-row x 128-byte box
  static constexpr int TILE_BYTES = KCH * CHUNK_BYTES;
  static constexpr int STAGES = TILE_BYTES == 2 * CHUNK_BYTES ? 4 : 8;  // K/V ring slots (128 KB)
  static constexpr int SMEM_Q = 2 * TILE_BYTES;
  static constexpr int SMEM_RING = STAGES * TILE_BYTES;
  static constexpr int SMEM_BARS = 1024;
  static constexpr int SMEM_TOTAL = 1024 /*align slack*/ + SMEM_Q + SMEM_RING + SMEM_BARS;
  static constexpr int SMEM_SPARSE = kUnitQueue * kSparseSlotBytes;   // block-sparse instance only
  static constexpr int THREADS = 384;                // 2 softmax WGs + load/MMA WG
  // per-thread registers after reallocation: softmax warpgroups / load+MMA warpgroup.
  // 2*128*REGS_SOFTMAX + 128*REGS_OTHER must not exceed the block's launch registers
  // (384 * registers per thread); the host checks this before launching.
  static constexpr uint32_t REGS_SOFTMAX = 192;
  static constexpr uint32_t REGS_OTHER = 120;
  static constexpr uint32_t TMEM_COLS = 512;
  // tensor-memory column map: S_t at 128 t, O_t at 256 + D t, P_t over S_t (16-bit)
  __host__ __device__ static constexpr uint32_t S_COL(int t) { return 128u * t; }
  __host__ __device__ static constexpr uint32_t O_COL(int t) { return 256u + (uint32_t)D * t; }
  __host__ __device__ static constexpr uint32_t P_COL(int t) { return 128u * t; }
};

// Warp roles: warp 0 issues the MMAs, warp 1 the TMA loads, warps 4-11 are the two
// softmax warpgroups.
constexpr int kWarpMma = 0;
constexpr int kWarpLoad = 1;

constexpr float kRescaleThresh = 8.0f;   // log2 units: the reference moves past this (16-bit P)
// FP8 weights: p = 2^(x - m_ref + kFp8Offset), so a row's largest weights sit near the top of
// e4m3's range instead of at 1 (weights below 2^-10 of the top round to zero, and a long row
// can hold many of them); the reference then moves once the max passes it by kFp8Thresh,
// which keeps p <= 2^8.75 < 448.  O / l is unchanged, the LSE takes kFp8Offset off.
constexpr float kFp8Offset = 8.0f, kFp8Thresh = 0.75f;
constexpr int kPolyEvery = 4;            // full tiles: one exponential pair in kPolyEvery on the FMA pipe (0: none)
// The FP8 block-sparse instance runs many single-tile steps, where one softmax warpgroup has
// the MUFU to itself, on a softmax with fewer instructions per score: there the FMA-pipe
// share only costs issue slots (measured 4 % slower at one pair in four), so it takes none.
// (The 16-bit block-sparse instance keeps the dense share: with every block kept it gives the
// dense forward's bits.)
template <bool SPARSE, bool FP8>
__host__ __device__ constexpr int poly_every() { return (SPARSE && FP8) ? 0 : kPolyEvery; }

struct FwdParams {
  void* o;
  float* lse;
  int B, Sq, Sk, Hq, Hkv, causal;
  int n_qblk;        // ceil(Sq / 256)
  int n_units;       // B * Hq * n_qblk
  int kv_group;      // (batch, KV head) pairs per scheduling group (their K/V fit in L2)
  int band;          // query blocks per band (a band of one group fills about one round)
  float c2;          // scale * log2(e)
  unsigned int* work;  // [2] dynamic scheduling (the kernel's DYN instance): next unit to
                       // hand out past the first round, CTAs done fetching; zero at launch,
                       // zeroed again by the launch's last CTA
  // Packed variable-length sequences (null: the dense [B, S, H, D] layout).  Sequence b owns
  // query rows cu_q[b] .. cu_q[b+1]-1 of q/o [Sq, Hq, D] and key rows cu_k[b] .. cu_k[b+1]-1
  // of k/v [Sk, Hkv, D] (Sq, Sk: the packed totals); LSE is [Hq, Sq].  n_qblk covers
  // max_sq query rows per sequence.
  const int* cu_q;
  const int* cu_k;
  int max_sq;
  // Paged K/V for packed queries (block_table non-null; cu_k unused): k/v are caches
  // [num_pages, page_size, Hkv, D], sequence b's key t in page block_table[b * max_blocks +
  // t / page_size] at row t % page_size, its length seqlens_k[b] (clamped to the table);
  // page_size a multiple of 128, so a K/V tile never crosses a page.
  const int* block_table;
  const int* seqlens_k;
  int max_blocks, page_size;
  // Block-sparse (the kernel's SPARSE instance): unit records of sp_stride uint16 each,
  // record (b * Hq + h) * n_qblk + query block.
  const uint16_t* sp;
  int sp_stride;
  float o_mul;          // O scale in the epilogue: the V descale of the FP8 instance, else 1
};

struct UnitInfo {
  int b, h, kvh, q0;         // q0: first query row of the unit within its sequence
  int sq, sk;                // the sequence's query and key lengths
  int qbase, kbase, mb;      // its first query / key row and batch index in the TMA maps
  int nkv[2];                // K/V tiles needed by Q tile 0 / 1 (0: tile has no work)
  int nkv_max;               // K/V steps of the unit (block-sparse: its list length)
  const uint16_t* ent;       // block-sparse: the unit's list in shared memory
};

__device__ __forceinline__ int fwd_kv_tiles(int sq, int sk, int causal, int r0) {
  if (r0 >= sq) return 0;
  int kend = sk;
  if (causal) {
    int rmax = min(r0 + 127, sq - 1);
    kend = min(sk, rmax + sk - sq + 1);
  }
  return kend > 0 ? (kend + 127) / 128 : 0;
}

// Packed sequences: the offsets must run forward inside the buffers and no sequence may
// be longer than max_sq.  The producer warps check them (each CTA a share) and record a
// status code for the first violation; the kernel itself clamps (fwd_unit), so bad offsets
// only shorten or empty a sequence.
__device__ __forceinline__ void fwd_check_lengths(const FwdParams& p, int lane, int cta, int ncta) {
  for (int b = cta * 32 + lane; b < p.B; b += ncta * 32) {
    const int q0 = __ldg(p.cu_q + b), q1 = __ldg(p.cu_q + b + 1);
    const int k0 = p.block_table ? 0 : __ldg(p.cu_k + b), k1 = p.block_table ? 0 : __ldg(p.cu_k + b + 1);  // paged: no cu_k
    if (q0 < 0 || q1 < q0 || q1 > p.Sq || q1 - q0 > p.max_sq || k0 < 0 || k1 < k0 || k1 > p.Sk)
      record_status(kStatusBadLengths, b);
  }
}

// Unit order.  The query blocks are cut into bands of `band` blocks, longest first; within
// a band, the (batch, KV head) pairs go in groups of kv_group, and within a group, query
// block descending, then the group's query heads.  The host sizes a group so its K and V
// fit in half the L2 and a (band, group) block fills about one round of the persistent
// grid: the CTAs in flight then share K/V tiles through L2, and consecutive rounds hold
// units of similar lengths (longest first overall, so the last units handed out are short).
// PACKED: the instance may see packed sequences -- the dynamic one; the static instance
// never does, and carries none of that code.  PAGED: the paged-cache instance (keys from
// seqlens_k and the block table instead of cu_k).
template <bool PACKED, bool PAGED = false>
__device__ __forceinline__ UnitInfo fwd_unit(const FwdParams& p, int u) {
  UnitInfo x;
  const int G = p.Hq / p.Hkv;
  const int n_bk = p.B * p.Hkv;
  const int per_band = p.band * p.B * p.Hq;            // units of a full band
  const int bi = u / per_band;
  const int bs = min(p.band, p.n_qblk - bi * p.band);  // this band's query blocks
  const int r = u - bi * per_band;
  const int full_grp = p.kv_group * G * bs;            // units of a full group in this band
  const int g = r / full_grp;
  const int gsize = min(p.kv_group, n_bk - g * p.kv_group);
  const int rr = r - g * full_grp;
  const int qb = p.n_qblk - 1 - (bi * p.band + rr / (gsize * G));
  const int rem = rr % (gsize * G);
  const int bk = g * p.kv_group + rem / G;
  x.b = bk / p.Hkv;
  x.kvh = bk % p.Hkv;
  x.h = x.kvh * G + rem % G;
  x.q0 = qb * 256;
  if (PACKED && p.cu_q) {
    // clamped into the buffers: offsets that run backwards or past the end give an empty
    // or shortened sequence, never an access outside q/k/v/o
    const int q_lo = min(max(__ldg(p.cu_q + x.b), 0), p.Sq);
    const int q_hi = min(max(__ldg(p.cu_q + x.b + 1), q_lo), p.Sq);
    // paged: keys 0 .. seqlens_k[b]-1 of the sequence's pages (p.Sk = the table's capacity)
    const int k_lo = PAGED ? 0 : min(max(__ldg(p.cu_k + x.b), 0), p.Sk);
    const int k_hi = PAGED ? min(max(__ldg(p.seqlens_k + x.b), 0), p.Sk)
                           : min(max(__ldg(p.cu_k + x.b + 1), k_lo), p.Sk);
    x.sq = q_hi - q_lo; x.sk = k_hi - k_lo;
    x.qbase = q_lo; x.kbase = k_lo; x.mb = 0;
  } else {
    x.sq = p.Sq; x.sk = p.Sk;
    x.qbase = 0; x.kbase = 0; x.mb = x.b;
  }
  x.nkv[0] = fwd_kv_tiles(x.sq, x.sk, p.causal, x.q0);
  x.nkv[1] = fwd_kv_tiles(x.sq, x.sk, p.causal, x.q0 + 128);
  x.nkv_max = max(x.nkv[0], x.nkv[1]);
  return x;
}

// Units are handed out in list order (longest first).  Static: round r gives CTA c unit
// r * ncta + c, reversed on odd rounds (a snake, so a CTA's long and short units pair up).
// Dynamic: CTA c starts with unit c, then its load warp takes the next unit from a global
// counter when it is ready for one (the kernel's DYN instance).  The host picks dynamic when
// its estimate of the static order's imbalance is large (few rounds of very different
// lengths); where the static order balances, the static instance measured faster.
__device__ __forceinline__ int fwd_unit_of(int round, int cta, int ncta) {
  return round * ncta + ((round & 1) ? (ncta - 1 - cta) : cta);
}
// Shared-memory map: Q tiles, K/V ring, then the barriers and two words.
template <int D, bool FP8 = false>
struct FwdSmem {
  using Cfg = FwdCfg<D, FP8>;
  uint8_t* q;          // [2][TILE]
  uint8_t* ring;       // [STAGES][TILE]
  uint64_t* kv_full;   // [STAGES]
  uint64_t* kv_empty;  // [STAGES]
  uint64_t* q_full;    // [2]
  uint64_t* q_empty;   // [2]
  uint64_t* s_full;    // [2]  S_t written (tcgen05.commit)
  uint64_t* p_full;    // [2]  P_t written and O_t rescaled (128 softmax threads)
  uint64_t* o_done;    // [2]  P_t V complete (tcgen05.commit)
  uint64_t* fin;       // [1]  every MMA of this CTA complete
  uint64_t* p_part;    // [2]  first 96 keys of P_t written, O_t rescaled (128 threads)
  uint32_t* tmem_holder;
  volatile int* abort_flag;
  uint64_t* unit_full;   // [kUnitQueue]  unit index written by the load warp
  uint64_t* unit_empty;  // [kUnitQueue]  read by the MMA warp and the 8 softmax warps
  volatile int* uq;      // [kUnitQueue]  the unit indices
  uint8_t* lists;        // [kUnitQueue][kSparseSlotBytes]  block-sparse unit records
  __device__ explicit FwdSmem(uint8_t* s) {
    q = s;
    ring = s + Cfg::SMEM_Q;
    uint64_t* b = (uint64_t*)(s + Cfg::SMEM_Q + Cfg::SMEM_RING);
    kv_full = b;
    kv_empty = b + Cfg::STAGES;
    q_full = b + 2 * Cfg::STAGES;
    q_empty = q_full + 2;
    s_full = q_full + 4;
    p_full = q_full + 6;
    o_done = q_full + 8;
    fin = q_full + 10;
    p_part = q_full + 11;
    tmem_holder = (uint32_t*)(q_full + 13);
    abort_flag = (volatile int*)(tmem_holder + 1);
    unit_full = q_full + 14;
    unit_empty = unit_full + kUnitQueue;
    uq = (volatile int*)(unit_empty + kUnitQueue);
    lists = s + Cfg::SMEM_Q + Cfg::SMEM_RING + Cfg::SMEM_BARS;
  }
};

// The n-th unit of this CTA, for a consuming warp: wait for the load warp to post it, read
// it, release the queue slot (one arrival per warp) unless the unit's shared-memory record
// is still needed (block-sparse: released by fwd_release_unit at the unit's end).
// Returns -1 if the wait gave up.
template <class SM>
__device__ __forceinline__ int fwd_next_unit(const SM& sm, int n, int where, bool release = true) {
  const int slot = n % kUnitQueue;
  if (!mbar_wait_warp(&sm.unit_full[slot], (n / kUnitQueue) & 1, sm.abort_flag, where)) return -1;
  const int u = sm.uq[slot];
  if (release) mbar_arrive_warp(&sm.unit_empty[slot]);
  return u;
}

template <class SM>
__device__ __forceinline__ void fwd_release_unit(const SM& sm, int n) {
  mbar_arrive_warp(&sm.unit_empty[n % kUnitQueue]);
}

// Block-sparse: the record of unit x (global, in the caller's workspace) and its copy in
// queue slot `slot` (shared memory), which sets the unit's step counts and list.
__device__ __forceinline__ const uint16_t* fwd_sparse_record(const FwdParams& p, const UnitInfo& x) {
  return p.sp + ((size_t)(x.b * p.Hq + x.h) * p.n_qblk + x.q0 / 256) * p.sp_stride;
}
template <class SM>
__device__ __forceinline__ void fwd_sparse_attach(const SM& sm, int slot, UnitInfo& x) {
  const uint16_t* rec = reinterpret_cast<const uint16_t*>(sm.lists + slot * kSparseSlotBytes);
  x.nkv_max = rec[0];
  x.nkv[0] = rec[1];
  x.nkv[1] = rec[2];
  x.ent = rec + 8;
}

// ------------------------------------------------------------------ TMA producer
template <int D, bool BF16, bool DYN, bool SPARSE, bool FP8, bool PAGED>
__device__ __forceinline__ void fwd_producer(const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                                             const CUtensorMap* tm_v, const FwdParams& p,
                                             const FwdSmem<D, FP8>& sm, int lane, int cta, int ncta) {
  using Cfg = FwdCfg<D, FP8>;
  if (lane == 0) {
    int slot = 0, ring_n = 0;            // ring position and total loads issued
    int q_load0 = 0, q_load1 = 0;        // Q tile loads issued
    int copy_n = -1;                     // block-sparse: unit whose record copy is in flight
    bool ok = true;
    for (int n = 0; ok; ++n) {
      // ---- the next unit (an index past the list ends the CTA), posted to the other roles
      int u;
      UnitInfo x;
      bool have_x = false;
      const int us = n % kUnitQueue;
      if (!DYN) {
        u = fwd_unit_of(n, cta, ncta);       // every role computes the same index
      } else {
        u = n == 0 ? cta : ncta + (int)atomicAdd(p.work, 1u);
        if (!SPARSE && p.cu_q) {
          // packed sequences shorter than the longest leave units without a single row
          // (nothing to compute or write): take the next one instead of handing them out
          for (; u < p.n_units; u = ncta + (int)atomicAdd(p.work, 1u)) {
            x = fwd_unit<DYN, PAGED>(p, u);
            if (x.q0 < x.sq) { have_x = true; break; }
          }
        }
        if (n >= kUnitQueue) {
          ok = mbar_wait(&sm.unit_empty[us], ((n / kUnitQueue) - 1) & 1, sm.abort_flag, 5);
          if (!ok) break;
        }
        sm.uq[us] = u;
        if (SPARSE && u < p.n_units) {
          // the unit's K/V tile list lands in the queue slot with the posting itself
          x = fwd_unit<DYN, PAGED>(p, u);
          const uint32_t bytes = (uint32_t)p.sp_stride * 2u;
          mbar_arrive_expect_tx(&sm.unit_full[us], bytes);
          bulk_copy_g2s(sm.lists + us * kSparseSlotBytes, fwd_sparse_record(p, x), bytes, &sm.unit_full[us]);
          copy_n = n;
          ok = mbar_wait(&sm.unit_full[us], (n / kUnitQueue) & 1, sm.abort_flag, 6);
          if (!ok) break;
          copy_n = -1;
          fwd_sparse_attach(sm, us, x);
        } else {
          mbar_arrive(&sm.unit_full[us]);
        }
      }
      if (u >= p.n_units) break;
      // (dynamic order: the unit's coordinates from the posted index, read back, so that their
      // arithmetic cannot be scheduled ahead of the posting the other roles wait for)
      if (!SPARSE && !have_x) x = fwd_unit<DYN, PAGED>(p, DYN ? (int)sm.uq[us] : u);
      for (int j = 0; j < x.nkv_max && ok; ++j) {
        const int kt = SPARSE ? (int)(x.ent[j] & 0x3fffu) : j;   // key tile of this step
        for (int kv = 0; kv < 2 && ok; ++kv) {
          if (ring_n >= Cfg::STAGES) {
            ok = mbar_wait(&sm.kv_empty[slot], ((ring_n / Cfg::STAGES) - 1) & 1, sm.abort_flag, 1);
            if (!ok) break;
          }
          uint8_t* dst = sm.ring + slot * Cfg::TILE_BYTES;
          mbar_arrive_expect_tx(&sm.kv_full[slot], Cfg::TILE_BYTES);
          const CUtensorMap* tm = kv ? tm_v : tm_k;
          {
            // K/V tile coordinates: (key row, batch), or for a paged cache (row in page, page);
            // a table entry outside the cache reads zeros (TMA fill), never other memory
            int krow = x.kbase + kt * 128, kouter = x.mb;
            if (PAGED) {
              krow = (kt * 128) % p.page_size;
              kouter = __ldg(p.block_table + (size_t)x.b * p.max_blocks + (kt * 128) / p.page_size);
            }
#pragma unroll
            for (int c = 0; c < Cfg::KCH; ++c)
              tma_load_4d(dst + c * Cfg::CHUNK_BYTES, tm, &sm.kv_full[slot], c * Cfg::CHUNK_ELEMS, x.kvh, krow,
                          kouter);
          }
          ++ring_n;
          slot = (slot + 1 == Cfg::STAGES) ? 0 : slot + 1;
          if (j == 0 && kv == 0) {
            // Q tiles after the first K tile, so K0 is in flight while Q waits for its slot
            for (int t = 0; t < 2 && ok; ++t) {
              if (x.nkv[t] == 0) continue;
              int& ql = t ? q_load1 : q_load0;
              if (ql > 0) {
                ok = mbar_wait(&sm.q_empty[t], (ql - 1) & 1, sm.abort_flag, 2);
                if (!ok) break;
              }
              uint8_t* qd = sm.q + t * Cfg::TILE_BYTES;
              mbar_arrive_expect_tx(&sm.q_full[t], Cfg::TILE_BYTES);
#pragma unroll
              for (int c = 0; c < Cfg::KCH; ++c)
                tma_load_4d(qd + c * Cfg::CHUNK_BYTES, tm_q, &sm.q_full[t], c * Cfg::CHUNK_ELEMS, x.h,
                            x.qbase + x.q0 + t * 128, x.mb);
              ++ql;
            }
          }
        }
      }
    }
    if (!ok) {
      // drain: every load issued must land before the CTA's shared memory goes away
      // (each slot's most recent load is among the last STAGES issued)
      int first = ring_n > Cfg::STAGES ? ring_n - Cfg::STAGES : 0;
      for (int n = first; n < ring_n; ++n)
        mbar_wait(&sm.kv_full[n % Cfg::STAGES], (n / Cfg::STAGES) & 1, nullptr, 3);
      if (q_load0 > 0) mbar_wait(&sm.q_full[0], (q_load0 - 1) & 1, nullptr, 4);
      if (q_load1 > 0) mbar_wait(&sm.q_full[1], (q_load1 - 1) & 1, nullptr, 4);
      if (SPARSE && copy_n >= 0)
        mbar_wait(&sm.unit_full[copy_n % kUnitQueue], (copy_n / kUnitQueue) & 1, nullptr, 7);
    }
    // this CTA takes no more units; the last CTA to get here zeroes the launch's counters
    // for the next launch that uses them (nothing reads them after this point)
    if (DYN && atomicAdd(p.work + 1, 1u) == (unsigned)ncta - 1) {
      atomicExch(p.work, 0u);
      atomicExch(p.work + 1, 0u);
    }
  }
  __syncwarp();
}

// ------------------------------------------------------------------ MMA issuer
// 4 k-steps of a shared x shared product along one 128-byte row: kind::f16 (16 elements a
// step) or, for FP8, kind::f8f6f4 (32 e4m3 elements a step); both step 32 bytes.
template <bool FP8>
__device__ __forceinline__ void qk_mma_x4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t acc_first) {
  if constexpr (!FP8) {
    mma_ss_x4(d_tmem, a_desc, b_desc, idesc, acc_first);
  } else {
    asm volatile(
        "{\n .reg .pred e, p, q;\n .reg .b32 r;\n .reg .b64 a, b;\n"
        " elect.sync r|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n setp.ne.b32 q, %5, 0;\n"
        " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n"
        " add.s64 a, %1, 2;\n add.s64 b, %2, 2;\n"
        " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %3, q;\n"
        " add.s64 a, %1, 4;\n add.s64 b, %2, 4;\n"
        " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %3, q;\n"
        " add.s64 a, %1, 6;\n add.s64 b, %2, 6;\n"
        " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %3, q;\n}\n"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc_first), "r"(1u) : "memory");
  }
}
// kind::f8f6f4 with A (e4m3 P) in tensor memory: a k-step is 32 keys = 8 columns of 4
// values; B (V, MN-major) steps 32 rows of 128 bytes (4096 bytes).  x3: keys 0-95, x1: one step.
__device__ __forceinline__ void mma_ts_f8_x3(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t acc_first) {
  asm volatile(
      "{\n .reg .pred e, p, q;\n .reg .b32 r, a;\n .reg .b64 b;\n"
      " elect.sync r|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n setp.ne.b32 q, %5, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n"
      " add.u32 a, %1, 8;\n add.s64 b, %2, 256;\n"
      " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [a], b, %3, q;\n"
      " add.u32 a, %1, 16;\n add.s64 b, %2, 512;\n"
      " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [a], b, %3, q;\n}\n"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(acc_first), "r"(1u) : "memory");
}
__device__ __forceinline__ void mma_ts_f8_x1(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t acc) {
  asm volatile(
      "{\n .reg .pred e, p;\n .reg .b32 r;\n"
      " elect.sync r|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n}\n"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(acc) : "memory");
}

template <int D, bool BF16, bool DYN, bool SPARSE, bool FP8, bool PAGED>
__device__ __forceinline__ void fwd_mma(const FwdParams& p, const FwdSmem<D, FP8>& sm, uint32_t tmem_base,
                                        int lane, int cta, int ncta) {
  using Cfg = FwdCfg<D, FP8>;
  (void)lane;
  {
    // (e4m3 is format 0 of kind::f8f6f4, in the same descriptor fields)
    constexpr uint32_t IDESC_QK = idesc_f16((BF16 && !FP8) ? 1 : 0, 128, 128, 0, 0);
    constexpr uint32_t IDESC_PV = idesc_f16((BF16 && !FP8) ? 1 : 0, 128, D, 0, 1);
    const uint32_t sQ_addr = smem_u32(sm.q);
    const uint32_t sRing_addr = smem_u32(sm.ring);
    int ring_n = 0;                       // ring position of this unit's first K tile
    int q_use0 = 0, q_use1 = 0;           // Q tile loads consumed (q_full phases)
    int pv0 = 0, pv1 = 0;                 // P_t V products issued (p_full phases)
    bool ok = true;
    auto issue_qk = [&](int t, uint32_t k_addr) {
      const uint32_t q_addr = sQ_addr + t * Cfg::TILE_BYTES;
      // D / 16 k-steps: 4 per 64-element (128-byte) chunk of the head dimension
#pragma unroll
      for (int c = 0; c < Cfg::KCH; ++c)
        qk_mma_x4<FP8>(tmem_base + Cfg::S_COL(t), smem_desc_sw128(q_addr + c * Cfg::CHUNK_BYTES, 16, 1024),
                       smem_desc_sw128(k_addr + c * Cfg::CHUNK_BYTES, 16, 1024), IDESC_QK, c > 0);
      mma_commit_warp(&sm.s_full[t]);
    };
    // Issue order per K/V step j:  PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1).
    // P_t lives in S_t's tensor-memory columns; QK_t(j+1) overwrites them right after
    // PV_t(j) read them.  tcgen05.mma instructions issued by one thread execute in
    // issue order, so the overwrite cannot overtake the read, and each softmax
    // warpgroup gets the other tile's PV + QK as cover for its exponentials.
    for (int n = 0; ok; ++n) {
      const int u = DYN ? fwd_next_unit(sm, n, 12, !SPARSE) : fwd_unit_of(n, cta, ncta);
      if (u < 0) { ok = false; break; }
      if (u >= p.n_units) break;
      UnitInfo x = fwd_unit<DYN, PAGED>(p, u);
      if (SPARSE) fwd_sparse_attach(sm, n % kUnitQueue, x);
      if (x.nkv_max == 0) {
        if (SPARSE) fwd_release_unit(sm, n);
        continue;
      }
      // whether Q tile t multiplies the K/V of step j: every step below its count (dense),
      // the steps whose list entry carries its bit (block-sparse)
      auto act = [&](int t, int j) -> bool {
        if constexpr (SPARSE) return j < x.nkv_max && ((x.ent[j] >> (14 + t)) & 1u);
        else return j < x.nkv[t];
      };
      int npv[2] = {0, 0};                     // block-sparse: P_t V products of this unit
      bool q_wait[2] = {true, true};           // block-sparse: Q_t not yet waited for
      const int base = ring_n;                 // K(j) at base + 2j, V(j) at base + 2j + 1
      // ---- prologue: S_t = Q_t K_0^T
      {
        const int pos = base;
        ok = mbar_wait_warp(&sm.kv_full[pos % Cfg::STAGES], (pos / Cfg::STAGES) & 1, sm.abort_flag, 10);
        if (!ok) break;
        const uint32_t k_addr = sRing_addr + (pos % Cfg::STAGES) * Cfg::TILE_BYTES;
        for (int t = 0; t < 2 && ok; ++t) {
          if (!act(t, 0)) continue;
          ok = mbar_wait_warp(&sm.q_full[t], (t ? q_use1 : q_use0) & 1, sm.abort_flag, 11);
          if (!ok) break;
          q_wait[t] = false;
          tc_fence_after();
          issue_qk(t, k_addr);
        }
        if (!ok) break;
        mma_commit_warp(&sm.kv_empty[pos % Cfg::STAGES]);
      }
      for (int j = 0; j < x.nkv_max && ok; ++j) {
        const int vpos = base + 2 * j + 1, kpos = base + 2 * j + 2;
        ok = mbar_wait_warp(&sm.kv_full[vpos % Cfg::STAGES], (vpos / Cfg::STAGES) & 1, sm.abort_flag, 13);
        if (!ok) break;
        const uint32_t v_addr = sRing_addr + (vpos % Cfg::STAGES) * Cfg::TILE_BYTES;
        const uint32_t k_addr = sRing_addr + (kpos % Cfg::STAGES) * Cfg::TILE_BYTES;
        bool k_ready = false;
        bool s_ahead[2] = {false, false};
        if (SPARSE && FP8 && j + 1 < x.nkv_max) {
          // FP8 block-sparse (8-slot ring of 16 KB tiles): a Q tile idle at this step but
          // working at the next one gets its next S now, ahead of the other tile's P V, so that
          // with alternating single-tile steps the two softmax warpgroups overlap -- only if
          // K_{j+1} (and that tile's Q) have landed: waiting here would hold up that P V.
          // (K_{j+1}'s slot held a tile of an earlier step, already waited for, so the parity
          // test sees no older phase.)
          for (int t = 0; t < 2; ++t) {
            if (act(t, j) || !act(t, j + 1)) continue;
            if (!k_ready)
              k_ready = __all_sync(0xffffffffu, mbar_try_wait(&sm.kv_full[kpos % Cfg::STAGES], (kpos / Cfg::STAGES) & 1));
            if (!k_ready) break;
            if (q_wait[t]) continue;
            tc_fence_after();
            issue_qk(t, k_addr);
            s_ahead[t] = true;
          }
        }
        for (int t = 0; t < 2; ++t) {
          const bool live = SPARSE || j < x.nkv[t];
          if (live && act(t, j)) {
            // ---- O_t += P_t V_j: keys 0-95 as soon as their P is written, then 96-127
            ok = mbar_wait_warp(&sm.p_part[t], (t ? pv1 : pv0) & 1, sm.abort_flag, 17);
            if (!ok) break;
            tc_fence_after();
            const uint32_t acc = SPARSE ? (npv[t] > 0 ? 1u : 0u) : (j > 0 ? 1u : 0u);
            if (FP8)   // keys 0-95: three k-steps of 32 (8 columns of 4 e4m3 P values, 32 V rows each)
              mma_ts_f8_x3(tmem_base + Cfg::O_COL(t), tmem_base + Cfg::P_COL(t),
                           smem_desc_sw128(v_addr, Cfg::CHUNK_BYTES, 1024), IDESC_PV, acc);
            else
              mma_ts_x6(tmem_base + Cfg::O_COL(t), tmem_base + Cfg::P_COL(t),
                        smem_desc_sw128(v_addr, Cfg::CHUNK_BYTES, 1024), IDESC_PV, acc);
            ok = mbar_wait_warp(&sm.p_full[t], (t ? pv1 : pv0) & 1, sm.abort_flag, 14);
            if (!ok) break;
            tc_fence_after();
            if (FP8)
              mma_ts_f8_x1(tmem_base + Cfg::O_COL(t), tmem_base + Cfg::P_COL(t) + 3 * 8,
                           smem_desc_sw128(v_addr + 3 * 4096, Cfg::CHUNK_BYTES, 1024), IDESC_PV, 1u);
            else
              mma_ts_x2(tmem_base + Cfg::O_COL(t), tmem_base + Cfg::P_COL(t) + 6 * 8,
                        smem_desc_sw128(v_addr + 6 * 2048, Cfg::CHUNK_BYTES, 1024), IDESC_PV, 1u);
            const bool last = SPARSE ? (++npv[t] == x.nkv[t]) : (j + 1 == x.nkv[t]);
            if (last) mma_commit_warp(&sm.o_done[t]);   // O_t complete for the epilogue
            if (t) ++pv1; else ++pv0;
          }
          // V_j's last reader is in the pipe: release its slot ahead of the second S
          if (t == 1) mma_commit_warp(&sm.kv_empty[vpos % Cfg::STAGES]);
          // ---- S_t = Q_t K_{j+1}^T
          if (live && act(t, j + 1) && !s_ahead[t]) {
            if (!k_ready) {
              ok = mbar_wait_warp(&sm.kv_full[kpos % Cfg::STAGES], (kpos / Cfg::STAGES) & 1, sm.abort_flag, 10);
              if (!ok) break;
              k_ready = true;
            }
            if (SPARSE && q_wait[t]) {
              // block-sparse: a Q tile whose first K/V step is not the unit's first
              ok = mbar_wait_warp(&sm.q_full[t], (t ? q_use1 : q_use0) & 1, sm.abort_flag, 11);
              if (!ok) break;
              q_wait[t] = false;
              tc_fence_after();
            }
            issue_qk(t, k_addr);
          }
        }
        if (!ok) break;
        if (j + 1 < x.nkv_max) {
          if (!k_ready) {
            // (cannot happen: the Q tile with the most K/V tiles needs K(j+1))
            ok = mbar_wait_warp(&sm.kv_full[kpos % Cfg::STAGES], (kpos / Cfg::STAGES) & 1, sm.abort_flag, 16);
            if (!ok) break;
          }
          mma_commit_warp(&sm.kv_empty[kpos % Cfg::STAGES]);
        }
      }
      if (!ok) break;
      ring_n = base + 2 * x.nkv_max;
      if (x.nkv[0] > 0) { mma_commit_warp(&sm.q_empty[0]); ++q_use0; }
      if (x.nkv[1] > 0) { mma_commit_warp(&sm.q_empty[1]); ++q_use1; }
      if (SPARSE) fwd_release_unit(sm, n);
    }
    // every MMA issued above completes before tensor memory is released
    mma_commit_warp(sm.fin);
    mbar_wait_warp(sm.fin, 0, nullptr, 15);
  }
  __syncwarp();
}

// ------------------------------------------------------------------ softmax + epilogue
// 2^x for a pair of finite x on the FMA pipe (the MUFU ex2 unit is the softmax's
// bottleneck: 16 results per clock per SM).  x = n + f with n = round(x) taken from the
// low mantissa bits of x + 1.5 * 2^23 and f in [-1/2, 1/2]; 2^f by a cubic fitted for
// minimum relative error on that interval (max 7.6e-5, below the 16-bit rounding of P);
// 2^n enters through the exponent field.  x is clamped at -125: the cubic's value lies in
// [0.7, 1.42), so with n >= -125 the exponent field stays >= 1 and the result normal (a
// clamped argument gives 2^-125, within 2^-125 of the true, smaller value).
__device__ __forceinline__ void exp2_poly_pair(float x0, float x1, float& a, float& b) {
  const f32x2 x = pack_f2(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const f32x2 t = add_f2(x, pack_f2(12582912.f, 12582912.f));       // 1.5 * 2^23 + n
  const f32x2 f = fma_f2(add_f2(t, pack_f2(-12582912.f, -12582912.f)), pack_f2(-1.f, -1.f), x);
  f32x2 q = fma_f2(pack_f2(0.055174146f, 0.055174146f), f, pack_f2(0.24261758f, 0.24261758f));
  q = fma_f2(q, f, pack_f2(0.69326109f, 0.69326109f));
  q = fma_f2(q, f, pack_f2(0.99992758f, 0.99992758f));
  float q0, q1, t0, t1;
  unpack_f2(q, q0, q1);
  unpack_f2(t, t0, t1);
  // n sits in the low bits of t; n << 23 added to the bits of 2^f scales it by 2^n
  a = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
  b = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
}

// Adds the two 16-bit values packed in pk (low half first) to two fp32 sums, one
// mixed-precision add each (no unpacking into fp32 registers).
template <bool BF16>
__device__ __forceinline__ void add_16x2_to_f32(uint32_t pk, float& lo, float& hi) {
  if (BF16)
    asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %2;\n add.rn.f32.bf16 %0, l, %0;\n add.rn.f32.bf16 %1, h, %1;\n}\n"
        : "+f"(lo), "+f"(hi) : "r"(pk));
  else
    asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %2;\n add.rn.f32.f16 %0, l, %0;\n add.rn.f32.f16 %1, h, %1;\n}\n"
        : "+f"(lo), "+f"(hi) : "r"(pk));
}

// One 32-key chunk of a row (v: the 32 scores as raw fp32 bits): p = 2^(scale2 * s - m) on
// pairs (one packed FMA per pair), P stored to tensor memory as 16-bit at taddr, both row
// sums (rse2: the fp32 weights, for the LSE; rs: the 16-bit weights the MMA multiplies, so
// O / l is an exact weighted average of V -- the largest weights' rounding cancels, which
// matters in rows one key dominates).  With POLY > 0, one pair in POLY is exponentiated
// by exp2_poly_pair (finite scores only).
template <bool BF16, int POLY>
__device__ __forceinline__ void softmax_chunk(const uint32_t (&v)[32], const f32x2 scale2,
                                              const f32x2 negm2, float (&rs)[4], f32x2 (&rse2)[2],
                                              const uint32_t taddr) {
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float x0, x1;
    unpack_f2(fma_f2(pack_f2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), scale2, negm2), x0, x1);
    float a, b2;
    if (POLY > 0 && (i % (POLY > 0 ? POLY : 1)) == POLY - 1) {
      exp2_poly_pair(x0, x1, a, b2);          // on the FMA pipe, sparing the MUFU
    } else {
      a = ex2(x0);
      b2 = ex2(x1);
    }
    rse2[i & 1] = add_f2(rse2[i & 1], pack_f2(a, b2));
    if (BF16) {
      __nv_bfloat162 h2 = __floats2bfloat162_rn(a, b2);
      pk[i] = *reinterpret_cast<uint32_t*>(&h2);
    } else {
      __half2 h2 = __floats2half2_rn(a, b2);
      pk[i] = *reinterpret_cast<uint32_t*>(&h2);
    }
    add_16x2_to_f32<BF16>(pk[i], rs[2 * (i & 1)], rs[2 * (i & 1) + 1]);
  }
  tmem_st16(taddr, pk);
}

// FP8 instance: the same chunk with P rounded to e4m3 (round to nearest even, saturating:
// p <= 2^8.75 under the offset reference, below e4m3's 448), 4 values per tensor-memory column
// (key 4j in the low byte of column j), 8 columns at taddr; rs sums the e4m3 values the
// MMA multiplies (each exact in f16, added to fp32 by mixed-precision adds).
template <int POLY>
__device__ __forceinline__ void softmax_chunk_fp8(const uint32_t (&v)[32], const f32x2 scale2,
                                                  const f32x2 negm2, float (&rs)[4], f32x2 (&rse2)[2],
                                                  const uint32_t taddr) {
  uint32_t pk[8];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float x0, x1;
    unpack_f2(fma_f2(pack_f2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), scale2, negm2), x0, x1);
    float a, b2;
    if (POLY > 0 && (i % (POLY > 0 ? POLY : 1)) == POLY - 1) {
      exp2_poly_pair(x0, x1, a, b2);
    } else {
      a = ex2(x0);
      b2 = ex2(x1);
    }
    rse2[i & 1] = add_f2(rse2[i & 1], pack_f2(a, b2));
    uint16_t e8;          // low byte: key 2i, high byte: key 2i + 1
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(e8) : "f"(b2), "f"(a));
    uint32_t h2;          // the two e4m3 values back as f16x2, for the row sum
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(e8));
    add_16x2_to_f32<false>(h2, rs[2 * (i & 1)], rs[2 * (i & 1) + 1]);
    if (i & 1) pk[i >> 1] |= (uint32_t)e8 << 16;
    else pk[i >> 1] = e8;
  }
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
               ::"r"(taddr), "r"(pk[0]), "r"(pk[1]), "r"(pk[2]), "r"(pk[3]), "r"(pk[4]), "r"(pk[5]),
                 "r"(pk[6]), "r"(pk[7])
               : "memory");
}

// rs (four fp32 chains) holds the sum of the weights the MMA multiplies (16-bit or e4m3).
template <bool BF16, bool FP8, int POLY>
__device__ __forceinline__ void softmax_chunk_any(const uint32_t (&v)[32], const f32x2 scale2, const f32x2 negm2,
                                                  float (&rs)[4], f32x2 (&rse2)[2], const uint32_t p_addr, int c) {
  if constexpr (FP8) softmax_chunk_fp8<POLY>(v, scale2, negm2, rs, rse2, p_addr + c * 8);
  else softmax_chunk<BF16, POLY>(v, scale2, negm2, rs, rse2, p_addr + c * 16);
}

__device__ __forceinline__ void sum_rounded(const float (&rs)[4], float& acc) {
  acc += (rs[0] + rs[1]) + (rs[2] + rs[3]);
}

// Running max over a 32-score chunk on 8 chains.
__device__ __forceinline__ void chunk_max(const uint32_t (&v)[32], float (&mx)[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k)
    mx[k] = max3f(mx[k], max3f(__uint_as_float(v[k]), __uint_as_float(v[k + 8]), __uint_as_float(v[k + 16])),
                  __uint_as_float(v[k + 24]));
}

__device__ __forceinline__ float max_of8(const float (&mx)[8]) {
  return fmaxf(max3f(mx[0], mx[1], mx[2]), max3f(max3f(mx[3], mx[4], mx[5]), mx[6], mx[7]));
}

// O_t row *= alpha, in place in tensor memory (32 columns at a time).
template <int D>
__device__ __forceinline__ void rescale_o_row(const uint32_t taddr, const float alpha) {
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(taddr + c * 32, r);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
    tmem_st32(taddr + c * 32, r);
  }
}

__device__ __forceinline__ void sum_f2x2(const f32x2 (&v)[2], float& acc) {
  float a0, a1;
  unpack_f2(add_f2(v[0], v[1]), a0, a1);
  acc += a0 + a1;
}

// Move the row's reference max to m_tile when it exceeds the reference by more than the
// instance's threshold, rescaling both sums and (after the first tile) the O_t row by
// 2^(m_ref - m_tile).  O_t holds P V up to the previous tile, complete: the commit that
// signalled this tile's S covers every earlier MMA.
template <int D, bool FP8>
__device__ __forceinline__ void move_reference(const float m_tile, const bool first, float& m_ref,
                                               float (&l_sum)[2], float (&l_lse)[2], const uint32_t o_addr) {
  const bool need = m_tile > m_ref + (FP8 ? kFp8Thresh : kRescaleThresh);
  float alpha = 1.f;
  if (need) {
    alpha = ex2(m_ref - m_tile);       // 0 when m_ref == -inf
    l_sum[0] *= alpha; l_sum[1] *= alpha;
    l_lse[0] *= alpha; l_lse[1] *= alpha;
    m_ref = m_tile;
  }
  if (!first && __any_sync(0xffffffffu, need)) rescale_o_row<D>(o_addr, alpha);
}

// A K/V tile every row of the Q tile sees in full, with scale >= 0 (the scale goes into
// the exponent's FMA).  Two passes over S: the row max from all 128 scores, then the
// exponentials.  P overwrites S columns 0-63 only, so the 16-bit instances' second pass
// holds chunks 0-1 from the first and loads chunks 2-3 again, which keeps a quarter fewer
// registers live through the exponentials (measured 2 % faster than holding all four);
// the FP8 instance, whose P takes only columns 0-31, holds all four (0.9 % faster than
// reloading).  The MMA warp may start on keys 0-95 at p_part.
template <int D, bool BF16, bool FP8, int POLY>
__device__ __forceinline__ void softmax_tile_full(const uint32_t s_addr, const uint32_t o_addr,
                                                  const uint32_t p_addr, const float c2, const bool first,
                                                  float& m_ref, float (&l_sum)[2], float (&l_lse)[2],
                                                  uint64_t* p_part) {
  constexpr bool RELOAD = !FP8;
  uint32_t v0[32], v1[32], v2[32], v3[32];
  float mx[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
  {
    tmem_ld32(s_addr, v0);
    tmem_ld32(s_addr + 32, v1);
    tmem_ld32(s_addr + 64, v2);
    tmem_ld32(s_addr + 96, v3);
    tmem_wait_ld_regs(v0);
    tmem_wait_ld_regs(v1);
    tmem_wait_ld_regs(v2);
    tmem_wait_ld_regs(v3);
    chunk_max(v0, mx);
    chunk_max(v1, mx);
    chunk_max(v2, mx);
    chunk_max(v3, mx);
  }
  move_reference<D, FP8>(max_of8(mx) * c2, first, m_ref, l_sum, l_lse, o_addr);
  const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
  const float nm = FP8 ? kFp8Offset - m_use : -m_use;
  const f32x2 scale2 = pack_f2(c2, c2), negm2 = pack_f2(nm, nm);
  // the row's sums are kept per key half (keys 0-63, 64-127) and added at the end, the order
  // the pair kernel's two half-row threads use, so both kernels give identical bits
  f32x2 rse2[2][2] = {{0ull, 0ull}, {0ull, 0ull}};
  float rs[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  if (RELOAD) tmem_ld32(s_addr + 64, v2);
  softmax_chunk_any<BF16, FP8, POLY>(v0, scale2, negm2, rs[0], rse2[0], p_addr, 0);
  softmax_chunk_any<BF16, FP8, POLY>(v1, scale2, negm2, rs[0], rse2[0], p_addr, 1);
  if (RELOAD) {
    tmem_wait_ld_regs(v2);
    tmem_ld32(s_addr + 96, v3);
  }
  softmax_chunk_any<BF16, FP8, POLY>(v2, scale2, negm2, rs[1], rse2[1], p_addr, 2);
  tmem_wait_st();
  tc_fence_before();
  mbar_arrive(p_part);
  if (RELOAD) tmem_wait_ld_regs(v3);
  softmax_chunk_any<BF16, FP8, POLY>(v3, scale2, negm2, rs[1], rse2[1], p_addr, 3);
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    sum_rounded(rs[hh], l_sum[hh]);
    sum_f2x2(rse2[hh], l_lse[hh]);
  }
}

// A tile that crosses the causal diagonal or the ragged end of K (or a negative scale):
// scores are scaled first and keys >= kl set to -inf, then max and exponentials.
template <int D, bool BF16, bool FP8>
__device__ __forceinline__ void softmax_tile_masked(const uint32_t s_addr, const uint32_t o_addr,
                                                    const uint32_t p_addr, const float c2, const int kl,
                                                    const bool first, float& m_ref, float (&l_sum)[2],
                                                    float (&l_lse)[2], uint64_t* p_part) {
  uint32_t v[4][32];
#pragma unroll
  for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, v[c]);
#pragma unroll
  for (int c = 0; c < 4; ++c) tmem_wait_ld_regs(v[c]);
  float mx[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      v[c][i] = __float_as_uint((c * 32 + i < kl) ? __uint_as_float(v[c][i]) * c2 : -INFINITY);
    chunk_max(v[c], mx);
  }
  move_reference<D, FP8>(max_of8(mx), first, m_ref, l_sum, l_lse, o_addr);
  const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
  const float nm = FP8 ? kFp8Offset - m_use : -m_use;
  const f32x2 scale2 = pack_f2(1.f, 1.f), negm2 = pack_f2(nm, nm);
  f32x2 rse2[2][2] = {{0ull, 0ull}, {0ull, 0ull}};
  float rs[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    softmax_chunk_any<BF16, FP8, 0>(v[c], scale2, negm2, rs[c >> 1], rse2[c >> 1], p_addr, c);
    if (c == 2) {
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_part);
    }
  }
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    sum_rounded(rs[hh], l_sum[hh]);
    sum_f2x2(rse2[hh], l_lse[hh]);
  }
}

template <int D, bool BF16, bool DYN, bool SPARSE, bool FP8, bool PAGED>
__device__ __forceinline__ void fwd_softmax(const FwdParams& p, const FwdSmem<D, FP8>& sm, uint32_t tmem_base,
                                            int warp, int lane, int cta, int ncta) {
  using Cfg = FwdCfg<D, FP8>;
  const int t = warp >> 2;                  // Q tile of this warpgroup (warp: 0-7 here)
  const int wl = warp & 3;                  // TMEM lane quarter (physical warp index % 4)
  const int row_in_tile = wl * 32 + lane;
  const uint32_t lane_addr = tmem_base + ((uint32_t)(wl * 32) << 16);
  const float c2 = p.c2;
  int s_n = 0, o_n = 0;                     // s_full / o_done phases consumed (o_done: one per unit)
  bool ok = true;
  for (int n = 0; ok; ++n) {
    const int u = DYN ? fwd_next_unit(sm, n, 23, !SPARSE) : fwd_unit_of(n, cta, ncta);
    if (u < 0) { ok = false; break; }
    if (u >= p.n_units) break;
    UnitInfo x = fwd_unit<DYN, PAGED>(p, u);
    if (SPARSE) fwd_sparse_attach(sm, n % kUnitQueue, x);
    const int nkv = x.nkv[t];
    const int row = x.q0 + t * 128 + row_in_tile;
    int klim = x.sk;
    if (p.causal) klim = min(x.sk, row + x.sk - x.sq + 1);
    // the first key tile that any row of this Q tile must mask
    const int r0 = x.q0 + t * 128;
    int kvis = x.sk;                        // keys every row of the tile can see
    if (p.causal) kvis = min(kvis, max(0, r0 + x.sk - x.sq + 1));
    const int mask_from = kvis / 128;
    // l_sum: sum of the rounded weights the MMA multiplied (normalises O); l_lse: sum of
    // the fp32 weights (gives the LSE without the rounding bias)
    float m_ref = -INFINITY, l_sum[2] = {0.f, 0.f}, l_lse[2] = {0.f, 0.f};
    const uint32_t s_addr = lane_addr + Cfg::S_COL(t), o_addr = lane_addr + Cfg::O_COL(t);
    const uint32_t p_addr = lane_addr + Cfg::P_COL(t);
    int i = 0;                              // block-sparse: this tile's K/V steps so far
    for (int j = 0; j < (SPARSE ? x.nkv_max : nkv); ++j) {
      int kt = j;                           // key tile of the step
      if constexpr (SPARSE) {
        const uint32_t e = x.ent[j];
        if (!((e >> (14 + t)) & 1u)) continue;
        kt = (int)(e & 0x3fffu);
      }
      const bool first = SPARSE ? (i == 0) : (j == 0);
      ok = mbar_wait_warp(&sm.s_full[t], s_n & 1, sm.abort_flag, 20 + t);
      if (!ok) break;
      ++s_n;
      tc_fence_after();
      if (kt < mask_from && c2 >= 0.f) {
        softmax_tile_full<D, BF16, FP8, poly_every<SPARSE, FP8>()>(s_addr, o_addr, p_addr, c2, first, m_ref, l_sum, l_lse,
                                                            &sm.p_part[t]);
      } else {
        const int kl = (kt >= mask_from) ? klim - kt * 128 : 128;   // keys >= kl: invisible to this row
        softmax_tile_masked<D, BF16, FP8>(s_addr, o_addr, p_addr, c2, kl, first, m_ref, l_sum, l_lse,
                                     &sm.p_part[t]);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full[t]);
      if (SPARSE) ++i;
    }
    if (!ok) break;
    // ---------------- epilogue: O / l, LSE
    if (nkv > 0) {
      ok = mbar_wait_warp(&sm.o_done[t], o_n & 1, sm.abort_flag, 22 + t);
      if (!ok) break;
      ++o_n;
      tc_fence_after();
    }
    const bool store = row < x.sq;
    const float L = l_sum[0] + l_sum[1], E = l_lse[0] + l_lse[1];
    const float inv_l = L > 0.f ? p.o_mul / L : 0.f;           // o_mul: FP8 V descale, else 1
    using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
    T* orow = reinterpret_cast<T*>(p.o) + (((size_t)x.mb * p.Sq + x.qbase + row) * p.Hq + x.h) * D;
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      uint32_t r[32];
      if (nkv > 0) {
        tmem_ld32(lane_addr + Cfg::O_COL(t) + c * 32, r);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = 0u;
      }
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float a = __uint_as_float(r[2 * i]) * inv_l, b2 = __uint_as_float(r[2 * i + 1]) * inv_l;
        if (BF16) {
          __nv_bfloat162 h2 = __floats2bfloat162_rn(a, b2);
          pk[i] = *reinterpret_cast<uint32_t*>(&h2);
        } else {
          __half2 h2 = __floats2half2_rn(a, b2);
          pk[i] = *reinterpret_cast<uint32_t*>(&h2);
        }
      }
      if (store) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
    }
    if (store && p.lse) {
      float lse = E > 0.f ? ((FP8 ? m_ref - kFp8Offset : m_ref) + __log2f(E)) * 0.69314718055994531f
                              : -INFINITY;
      p.lse[((size_t)x.mb * p.Hq + x.h) * p.Sq + x.qbase + row] = lse;
    }
    tc_fence_before();
    if (SPARSE) fwd_release_unit(sm, n);
  }
}

// Every role ends here: one block-wide named barrier (id 1, all 384 threads), then the
// warp that allocated tensor memory releases it.
__device__ __forceinline__ void fwd_teardown(bool owner, uint32_t tmem_base, uint32_t ncols) {
  tc_fence_before();
  asm volatile("bar.sync 1, 384;" ::: "memory");
  if (owner) {
    tc_fence_after();
    tmem_dealloc(tmem_base, ncols);
  }
}

template <int D, bool BF16, bool DYN, bool SPARSE, bool FP8 = false, bool PAGED = false>
__global__ void __launch_bounds__(384, 1)
attn_fwd_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using Cfg = FwdCfg<D, FP8>;
  static_assert(DYN || !SPARSE, "the block-sparse units go through the dynamic unit queue");
  static_assert(!FP8 || (BF16 && D == 128), "FP8: D = 128, bf16 output");
  static_assert(!PAGED || (DYN && !SPARSE && !FP8), "the paged instance: dynamic, dense blocks, 16-bit");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const FwdSmem<D, FP8> sm(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ncta = gridDim.x;
  const int cta = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < Cfg::STAGES; ++i) { mbar_init(&sm.kv_full[i], 1); mbar_init(&sm.kv_empty[i], 1); }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sm.q_full[t], 1); mbar_init(&sm.q_empty[t], 1);
      mbar_init(&sm.s_full[t], 1); mbar_init(&sm.p_full[t], 128); mbar_init(&sm.o_done[t], 1);
      mbar_init(&sm.p_part[t], 128);
    }
    mbar_init(sm.fin, 1);
    // unit queue: the load warp posts, the MMA warp and the 8 softmax warps each release
    for (int i = 0; i < kUnitQueue; ++i) { mbar_init(&sm.unit_full[i], 1); mbar_init(&sm.unit_empty[i], 9); }
    *sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(sm.tmem_holder, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == kWarpLoad && lane == 0) {
    tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *sm.tmem_holder;

  if (warp < 4) {
    // load / MMA warpgroup gives registers away; warp 2 checks packed sequence offsets,
    // warp 3 has no role
    regs_dec<Cfg::REGS_OTHER>();
    if (warp == kWarpLoad) fwd_producer<D, BF16, DYN, SPARSE, FP8, PAGED>(&tm_q, &tm_k, &tm_v, p, sm, lane, cta, ncta);
    else if (warp == kWarpMma) fwd_mma<D, BF16, DYN, SPARSE, FP8, PAGED>(p, sm, tmem_base, lane, cta, ncta);
    else if (warp == 2 && p.cu_q) fwd_check_lengths(p, lane, cta, ncta);
    fwd_teardown(warp == kWarpMma, tmem_base, Cfg::TMEM_COLS);
  } else {
    regs_inc<Cfg::REGS_SOFTMAX>();
    fwd_softmax<D, BF16, DYN, SPARSE, FP8, PAGED>(p, sm, tmem_base, warp - 4, lane, cta, ncta);
    fwd_teardown(false, tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace sa

