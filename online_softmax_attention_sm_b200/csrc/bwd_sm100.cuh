// bwd_sm100.cuh -- attention backward (dQ, dK, dV from dO) on sm_100a tensor cores.
//
// Method: the StreamAttention page's "Backward" (recompute the QK tiles from the saved LSE,
// stream dQ/dK/dV without materialising the attention matrix) and the flash-attn-volta
// page's backward.  With c2 = scale * log2(e) and lse2 = LSE * log2(e):
//   P  = 2^(c2 S - lse2)  (0 at invisible keys),   Delta = rowsum(dO * O),
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - Delta),  dQ = scale dS K,  dK = scale dS^T Q.
//
// B200 design: three kernels, no atomics.
//   * bwd_prep: -lse2 and -Delta per query row into the caller's workspace ([B, Hq, Sq_pad],
//     Sq_pad = Sq rounded up to 128; padding rows get -lse2 = -inf (P = 0) and -Delta = 0,
//     so a whole 128-row slice can always be copied); stored negated so that
//     c2 S - lse2 and dP - Delta are one packed FMA / ADD each;
//   * attn_bwd_kv<D>: one CTA per (128-key tile, KV head, batch) keeps K and V in shared
//     memory and walks every (query head of the group, 128-row Q tile) that sees the tile:
//     S^T = K Q^T and dP^T = V dO^T (tcgen05, both operands K-major from shared memory),
//     P^T and dS^T in registers (one key row per thread), written back to tensor memory as
//     16-bit, then dV += P^T dO and dK += dS^T Q (A from tensor memory, B = the Q / dO
//     tile read MN-major) -- dK and dV of a KV head accumulate over its query heads in
//     tensor memory;
//   * attn_bwd_q<D>: one CTA per (128-row Q tile, query head, batch) keeps Q and dO and
//     walks its K/V tiles: S = Q K^T, dP = dO V^T, P and dS per query row, dQ += dS K.
// dQ is recomputed apart from dK/dV (7 tile products instead of 5) so that no tile needs
// an atomic update and every product uses an operand form of the forward kernel.
//
// Each 128 x 128 step is split into two 64-column halves (queries in the KV kernel, keys
// in the Q kernel); softmax warpgroup c owns half c.  The MMA warp issues, per step n,
//   [half 0 done] dV/dK (or dQ) products of half 0 of step n, S/dP of half 0 of step n+1,
//   [half 1 done] products of half 1 of step n,               S/dP of half 1 of step n+1,
// so one warpgroup works while the tensor core runs the other's products (the forward's
// two-tile interleave).  A product reading 16-bit P / dS from tensor memory is issued
// before the S / dP of the next step that overwrites those columns; tcgen05.mma ops
// from one thread execute in order.
#pragma once
#include "ptx.cuh"
#include <cuda_fp16.h>
#include <cuda_bf16.h>

namespace sa {

template <int D>
struct BwdCfg {
  static constexpr int KCH = D / 64;                 // 128-byte chunks along D
  static constexpr int CHUNK = 128 * 128;            // one 128-row x 64-element box
  static constexpr int TILE = KCH * CHUNK;           // a 128 x D tile
  static constexpr int STAGES = 2;                   // ring slots (Q+dO or K+V pairs)
  static constexpr int VEC = 2 * 128 * 4;            // per-slot lse2 + Delta rows (KV kernel)
  static constexpr int SLOT = 2 * TILE + VEC;
  static constexpr int SMEM_BARS = 256;
  static constexpr int SMEM_TOTAL = 1024 + 2 * TILE + STAGES * SLOT + SMEM_BARS;
  static constexpr int THREADS = 384;                // MMA warp, load warp, 2 idle, 2 WGs
  static constexpr uint32_t TMEM_COLS = 512;
  // tensor-memory columns: S (or S^T) halves at 0 / 64, dP halves at 128 / 192 (fp32);
  // 16-bit P over the first 32 columns of its S half, dS likewise over dP;
  // accumulators: dV (or dQ) at 256, dK at 256 + D
  static constexpr uint32_t S_COL = 0, DP_COL = 128, ACC0 = 256, ACC1 = 256 + D;
};

struct BwdParams {
  const void* o;        // [B, Sq, Hq, D] forward output (prep)
  const void* dout;     // [B, Sq, Hq, D]
  const float* lse;     // [B, Hq, Sq] forward LSE (natural log)
  float* nlse2;         // [B, Hq, Sq_pad] workspace: -LSE * log2(e)
  float* ndelta;        // [B, Hq, Sq_pad] workspace: -rowsum(dO * O)
  void* dq;             // [B, Sq, Hq, D]
  void* dk;             // [B, Sk, Hkv, D]
  void* dv;             // [B, Sk, Hkv, D]
  int B, Sq, Sk, Hq, Hkv, G, causal, sq_pad, n_qt, n_kt;
  float c2, scale;
};

// ---------------------------------------------------------------- preprocess
// One thread per (batch, padded query row, query head), head fastest (the O / dO rows of
// consecutive threads are contiguous).
template <int D, bool BF16>
__global__ void __launch_bounds__(256) bwd_prep(const BwdParams p) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long n = (long long)p.B * p.sq_pad * p.Hq;
  if (i >= n) return;
  const int h = (int)(i % p.Hq);
  const long long bq = i / p.Hq;
  const int q = (int)(bq % p.sq_pad), b = (int)(bq / p.sq_pad);
  const size_t out = ((size_t)b * p.Hq + h) * p.sq_pad + q;
  if (q >= p.Sq) {
    p.nlse2[out] = -INFINITY;
    p.ndelta[out] = 0.f;
    return;
  }
  const size_t row = (((size_t)b * p.Sq + q) * p.Hq + h) * D;
  const uint4* o4 = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.o) + row);
  const uint4* d4 = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.dout) + row);
  uint4 ov[D / 8], dv[D / 8];
#pragma unroll
  for (int c = 0; c < D / 8; ++c) { ov[c] = o4[c]; dv[c] = d4[c]; }
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    const uint32_t* a = reinterpret_cast<const uint32_t*>(&ov[c]);
    const uint32_t* g = reinterpret_cast<const uint32_t*>(&dv[c]);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float a0, a1, g0, g1;
      if (BF16) {
        a0 = __uint_as_float(a[j] << 16); a1 = __uint_as_float(a[j] & 0xffff0000u);
        g0 = __uint_as_float(g[j] << 16); g1 = __uint_as_float(g[j] & 0xffff0000u);
      } else {
        const float2 fa = __half22float2(*reinterpret_cast<const __half2*>(&a[j]));
        const float2 fg = __half22float2(*reinterpret_cast<const __half2*>(&g[j]));
        a0 = fa.x; a1 = fa.y; g0 = fg.x; g1 = fg.y;
      }
      acc = fmaf(a0, g0, acc);
      acc = fmaf(a1, g1, acc);
    }
  }
  const float l = p.lse[((size_t)b * p.Hq + h) * p.Sq + q];
  p.nlse2[out] = -l * 1.4426950408889634f;    // row without keys: +inf, never unmasked
  p.ndelta[out] = -acc;
}

// ---------------------------------------------------------------- shared helpers
// 4 k-steps with A in tensor memory (16 elements = 8 columns of 16-bit pairs per step) and
// B stepping 16 rows of 128 bytes per step.
__device__ __forceinline__ void mma_ts_x4(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t acc_first) {
  asm volatile(
      "{\n .reg .pred e, p, q;\n .reg .b32 r, a;\n .reg .b64 b;\n"
      " elect.sync r|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n setp.ne.b32 q, %5, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n"
      " add.u32 a, %1, 8;\n add.s64 b, %2, 128;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, q;\n"
      " add.u32 a, %1, 16;\n add.s64 b, %2, 256;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, q;\n"
      " add.u32 a, %1, 24;\n add.s64 b, %2, 384;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [a], b, %3, q;\n}\n"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(acc_first), "r"(1u) : "memory");
}

__device__ __forceinline__ f32x2 mul_f2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 16-bit pair of two fp32 values (round to nearest even)
template <bool BF16>
__device__ __forceinline__ uint32_t bwd_pack(float lo, float hi) {
  if (BF16) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Tensor-memory loads / stores of 16 and 8 columns (32 lanes x 32-bit, one lane per thread).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
               ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
                 "r"(r[6]), "r"(r[7])
               : "memory");
}
// tcgen05.wait::ld naming the 32 registers of the loads it waits for (no use of them can be
// scheduled above it)
__device__ __forceinline__ void tmem_wait_ld_2x16(uint32_t (&a)[16], uint32_t (&b)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]), "+r"(a[6]),
                 "+r"(a[7]), "+r"(a[8]), "+r"(a[9]), "+r"(a[10]), "+r"(a[11]), "+r"(a[12]), "+r"(a[13]),
                 "+r"(a[14]), "+r"(a[15]), "+r"(b[0]), "+r"(b[1]), "+r"(b[2]), "+r"(b[3]), "+r"(b[4]),
                 "+r"(b[5]), "+r"(b[6]), "+r"(b[7]), "+r"(b[8]), "+r"(b[9]), "+r"(b[10]), "+r"(b[11]),
                 "+r"(b[12]), "+r"(b[13]), "+r"(b[14]), "+r"(b[15])
               :: "memory");
}

// P and dS of one 64-column half for the calling thread's row (S at s_addr, dP at dp_addr,
// fp32 columns).  nl(j), nd(j) = -lse2 and -Delta of columns (2j, 2j+1) as a packed pair;
// columns lo <= c < hi are visible (the rest get P = dS = 0).  P = 2^(c2 s - lse2) and
// dS = P (dP - Delta) on packed f32x2 pairs; dS (and, if STORE_P, P) go back as 16-bit pairs
// over the half's first 32 columns (pair j at column j).  Four 16-column pieces; the loads
// of a piece are issued before the arithmetic of the previous one.  A piece's 16-bit pairs
// land on columns whose fp32 values earlier pieces have already read.
template <bool BF16, bool STORE_P, typename NL, typename ND>
__device__ __forceinline__ void bwd_half(uint32_t s_addr, uint32_t dp_addr, f32x2 c2, NL nl, ND nd, int lo, int hi) {
  const bool full = lo <= 0 && hi >= 64;
  uint32_t sv[2][16], dv[2][16];
  tmem_ld16(s_addr, sv[0]);
  tmem_ld16(dp_addr, dv[0]);
  tmem_wait_ld_2x16(sv[0], dv[0]);
#pragma unroll
  for (int pc = 0; pc < 4; ++pc) {
    const int cur = pc & 1;
    if (pc + 1 < 4) {
      tmem_ld16(s_addr + 16 * (pc + 1), sv[cur ^ 1]);
      tmem_ld16(dp_addr + 16 * (pc + 1), dv[cur ^ 1]);
    }
    uint32_t pp[8], dsp[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int j = 8 * pc + i, c = 2 * j;        // pair j: columns c, c + 1 of the half
      float x0, x1;
      unpack_f2(fma_f2(pack_f2(__uint_as_float(sv[cur][2 * i]), __uint_as_float(sv[cur][2 * i + 1])), c2, nl(j)),
                x0, x1);
      float p0 = ex2(x0), p1 = ex2(x1);
      if (!full) {
        p0 = (c >= lo && c < hi) ? p0 : 0.f;
        p1 = (c + 1 >= lo && c + 1 < hi) ? p1 : 0.f;
      }
      const f32x2 d2 = mul_f2(pack_f2(p0, p1),
                              add_f2(pack_f2(__uint_as_float(dv[cur][2 * i]), __uint_as_float(dv[cur][2 * i + 1])),
                                     nd(j)));
      float d0, d1;
      unpack_f2(d2, d0, d1);
      if (STORE_P) pp[i] = bwd_pack<BF16>(p0, p1);
      dsp[i] = bwd_pack<BF16>(d0, d1);
    }
    if (STORE_P) tmem_st8(s_addr + 8 * pc, pp);
    tmem_st8(dp_addr + 8 * pc, dsp);
    if (pc + 1 < 4) tmem_wait_ld_2x16(sv[cur ^ 1], dv[cur ^ 1]);
  }
}

// Shared-memory map of both backward kernels: two fixed tiles (K, V or Q, dO), a ring of
// STAGES slots (Q, dO, lse2, Delta rows or K, V), barriers.
template <int D>
struct BwdSmem {
  using Cfg = BwdCfg<D>;
  uint8_t* fix0;
  uint8_t* fix1;
  uint8_t* ring;
  uint64_t* fix_full;     // [1]
  uint64_t* full;         // [STAGES]
  uint64_t* empty;        // [STAGES]
  uint64_t* s_ready;      // [2] S / dP half written (tcgen05.commit)
  uint64_t* p_ready;      // [2] P / dS half written (128 threads)
  uint64_t* fin;          // [1] every product issued has completed
  uint32_t* tmem_holder;
  volatile int* abort_flag;
  __device__ explicit BwdSmem(uint8_t* s) {
    fix0 = s;
    fix1 = s + Cfg::TILE;
    ring = s + 2 * Cfg::TILE;
    uint64_t* b = (uint64_t*)(ring + Cfg::STAGES * Cfg::SLOT);
    fix_full = b;
    full = b + 1;
    empty = full + Cfg::STAGES;
    s_ready = empty + Cfg::STAGES;
    p_ready = s_ready + 2;
    fin = p_ready + 2;
    tmem_holder = (uint32_t*)(fin + 1);
    abort_flag = (volatile int*)(tmem_holder + 1);
  }
  __device__ uint8_t* slot(int i) const { return ring + i * Cfg::SLOT; }
};

template <int D>
__device__ __forceinline__ void bwd_init(const BwdSmem<D>& sm) {
  mbar_init(sm.fix_full, 1);
  for (int i = 0; i < BwdCfg<D>::STAGES; ++i) { mbar_init(&sm.full[i], 1); mbar_init(&sm.empty[i], 1); }
  for (int i = 0; i < 2; ++i) { mbar_init(&sm.s_ready[i], 1); mbar_init(&sm.p_ready[i], 128); }
  mbar_init(sm.fin, 1);
  *sm.abort_flag = 0;
  fence_barrier_init();
}

// The MMA warp's loop shared by both kernels: nsteps steps, each two halves; issue_s(n, h)
// issues the S / dP products of half h of step n and commits s_ready[h]; issue_acc(n, h)
// the accumulating products of half h of step n.  Step n's ring slot is released once its
// accumulating products complete (not waiting for step n + 1's S / dP, so the load of step
// n + 2 starts a product earlier).  Returns false if a wait gave up.
template <int D, typename IssueS, typename IssueAcc>
__device__ __forceinline__ bool bwd_mma_loop(const BwdSmem<D>& sm, int nsteps, IssueS issue_s, IssueAcc issue_acc) {
  using Cfg = BwdCfg<D>;
  if (nsteps == 0) return true;
  if (!mbar_wait_warp(&sm.full[0], 0, sm.abort_flag, 60)) return false;
  tc_fence_after();
  issue_s(0, 0);
  issue_s(0, 1);
  for (int n = 0; n < nsteps; ++n) {
    const bool more = n + 1 < nsteps;
    for (int h = 0; h < 2; ++h) {
      if (!mbar_wait_warp(&sm.p_ready[h], n & 1, sm.abort_flag, 61 + h)) return false;
      tc_fence_after();
      issue_acc(n, h);
      // the slot's last reader is in the pipe: release it before step n + 1's second half
      if (h == 1) mma_commit_warp(&sm.empty[n % Cfg::STAGES]);
      if (more) {
        if (h == 0) {
          const int m = n + 1;
          if (!mbar_wait_warp(&sm.full[m % Cfg::STAGES], (m / Cfg::STAGES) & 1, sm.abort_flag, 63)) return false;
          tc_fence_after();
        }
        issue_s(n + 1, h);
      }
    }
  }
  return true;
}

// Every role ends here: one block-wide named barrier, then the allocating warp frees
// tensor memory.
__device__ __forceinline__ void bwd_teardown(bool owner, uint32_t tmem_base, uint32_t ncols) {
  tc_fence_before();
  asm volatile("bar.sync 1, 384;" ::: "memory");
  if (owner) {
    tc_fence_after();
    tmem_dealloc(tmem_base, ncols);
  }
}

// Producer drain after a failed wait: every load issued must land before shared memory
// goes away (loads of steps first .. issued-1 may be in flight).
template <int D>
__device__ __forceinline__ void bwd_drain(const BwdSmem<D>& sm, bool fix_issued, int issued) {
  using Cfg = BwdCfg<D>;
  if (fix_issued) mbar_wait(sm.fix_full, 0, nullptr, 69);
  for (int n = issued > Cfg::STAGES ? issued - Cfg::STAGES : 0; n < issued; ++n)
    mbar_wait(&sm.full[n % Cfg::STAGES], (n / Cfg::STAGES) & 1, nullptr, 69);
}

// 16-bit output row of D values from tensor memory columns col .. col + n - 1 (n = 32 or a
// multiple), times `mul`, stored to dst (if store).
template <bool BF16, int N>
__device__ __forceinline__ void bwd_store_row(uint32_t taddr, float mul, void* dst, bool store, bool zero) {
#pragma unroll 1
  for (int c = 0; c < N / 32; ++c) {
    uint32_t r[32];
    if (!zero) {
      tmem_ld32(taddr + c * 32, r);
      tmem_wait_ld_regs(r);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) r[i] = 0u;
    }
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      pk[i] = bwd_pack<BF16>(__uint_as_float(r[2 * i]) * mul, __uint_as_float(r[2 * i + 1]) * mul);
    if (store) {
      uint4* d4 = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(dst) + c * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
    }
  }
}

// ---------------------------------------------------------------- dK, dV
template <int D, bool BF16>
__global__ void __launch_bounds__(384, 1)
attn_bwd_kv(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
            const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
            const BwdParams p) {
  using Cfg = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const BwdSmem<D> sm(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // one flat grid, longest first: key tile major (causal: the first tiles see the most
  // queries), then batch, then KV head
  const int per_tile = p.Hkv * p.B;
  const int kt = (int)blockIdx.x / per_tile, b = ((int)blockIdx.x % per_tile) / p.Hkv, kvh = (int)blockIdx.x % p.Hkv;
  // query tiles that see this key tile: all, or (causal) from the first row whose
  // bottom-right-aligned diagonal reaches the tile's first key
  int qt0 = 0;
  if (p.causal) {
    const int need = kt * 128 - (p.Sk - p.Sq);     // first query row that sees key kt*128
    qt0 = need <= 0 ? 0 : need / 128;
  }
  const int per_head = qt0 < p.n_qt ? p.n_qt - qt0 : 0;
  const int nsteps = p.G * per_head;
  if (threadIdx.x == 0) bwd_init(sm);
  if (warp == 0) { tmem_alloc(sm.tmem_holder, Cfg::TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_holder;
  auto step_head = [&](int n) { return kvh * p.G + n / per_head; };
  auto step_qt = [&](int n) { return qt0 + n % per_head; };

  if (warp == 1) {
    // ---- loads: K and V once, then (Q, dO, lse2, Delta) per step
    if (lane == 0) {
      bool ok = true;
      int issued = 0;
      tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_do); tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_v);
      if (nsteps > 0) {                 // (no step: nothing waits for K and V, so none are loaded)
        mbar_arrive_expect_tx(sm.fix_full, 2 * Cfg::TILE);
        for (int c = 0; c < Cfg::KCH; ++c) {
          tma_load_4d(sm.fix0 + c * Cfg::CHUNK, &tm_k, sm.fix_full, c * 64, kvh, kt * 128, b);
          tma_load_4d(sm.fix1 + c * Cfg::CHUNK, &tm_v, sm.fix_full, c * 64, kvh, kt * 128, b);
        }
      }
      for (int n = 0; n < nsteps && ok; ++n) {
        const int s = n % Cfg::STAGES;
        if (n >= Cfg::STAGES) {
          ok = mbar_wait(&sm.empty[s], ((n / Cfg::STAGES) - 1) & 1, sm.abort_flag, 64);
          if (!ok) break;
        }
        const int h = step_head(n), qt = step_qt(n);
        uint8_t* dst = sm.slot(s);
        mbar_arrive_expect_tx(&sm.full[s], 2 * Cfg::TILE + Cfg::VEC);
        for (int c = 0; c < Cfg::KCH; ++c) {
          tma_load_4d(dst + c * Cfg::CHUNK, &tm_q, &sm.full[s], c * 64, h, qt * 128, b);
          tma_load_4d(dst + Cfg::TILE + c * Cfg::CHUNK, &tm_do, &sm.full[s], c * 64, h, qt * 128, b);
        }
        const size_t vrow = ((size_t)b * p.Hq + h) * p.sq_pad + (size_t)qt * 128;
        bulk_copy_g2s(dst + 2 * Cfg::TILE, p.nlse2 + vrow, 512, &sm.full[s]);
        bulk_copy_g2s(dst + 2 * Cfg::TILE + 512, p.ndelta + vrow, 512, &sm.full[s]);
        issued = n + 1;
      }
      if (!ok) bwd_drain(sm, nsteps > 0, issued);
    }
    __syncwarp();
    bwd_teardown(false, tmem, Cfg::TMEM_COLS);
  } else if (warp == 0) {
    // ---- MMA issue
    constexpr uint32_t IDESC_S = idesc_f16(BF16 ? 1 : 0, 128, 64, 0, 0);
    constexpr uint32_t IDESC_ACC = idesc_f16(BF16 ? 1 : 0, 128, D, 0, 1);
    const uint32_t k_addr = smem_u32(sm.fix0), v_addr = smem_u32(sm.fix1);
    bool ok = nsteps == 0 || mbar_wait_warp(sm.fix_full, 0, sm.abort_flag, 65);
    if (ok) {
      // S^T half h = K Q[h]^T, dP^T half h = V dO[h]^T  (M = 128 keys, N = 64 queries)
      auto issue_s = [&](int n, int h) {
        const uint32_t q_addr = smem_u32(sm.slot(n % Cfg::STAGES)), do_addr = q_addr + Cfg::TILE;
#pragma unroll
        for (int c = 0; c < Cfg::KCH; ++c)
          mma_ss_x4(tmem + Cfg::S_COL + 64 * h, smem_desc_sw128(k_addr + c * Cfg::CHUNK, 16, 1024),
                    smem_desc_sw128(q_addr + c * Cfg::CHUNK + h * 8192, 16, 1024), IDESC_S, c > 0);
#pragma unroll
        for (int c = 0; c < Cfg::KCH; ++c)
          mma_ss_x4(tmem + Cfg::DP_COL + 64 * h, smem_desc_sw128(v_addr + c * Cfg::CHUNK, 16, 1024),
                    smem_desc_sw128(do_addr + c * Cfg::CHUNK + h * 8192, 16, 1024), IDESC_S, c > 0);
        mma_commit_warp(&sm.s_ready[h]);
      };
      // dV += P^T[h] dO[h], dK += dS^T[h] Q[h]  (K = the half's 64 queries)
      auto issue_acc = [&](int n, int h) {
        const uint32_t q_addr = smem_u32(sm.slot(n % Cfg::STAGES)), do_addr = q_addr + Cfg::TILE;
        const uint32_t acc = (n > 0 || h > 0) ? 1u : 0u;
        mma_ts_x4(tmem + Cfg::ACC0, tmem + Cfg::S_COL + 64 * h,
                  smem_desc_sw128(do_addr + h * 8192, Cfg::CHUNK, 1024), IDESC_ACC, acc);
        mma_ts_x4(tmem + Cfg::ACC1, tmem + Cfg::DP_COL + 64 * h,
                  smem_desc_sw128(q_addr + h * 8192, Cfg::CHUNK, 1024), IDESC_ACC, acc);
      };
      ok = bwd_mma_loop<D>(sm, nsteps, issue_s, issue_acc);
    }
    if (!ok) *sm.abort_flag = 1;
    mma_commit_warp(sm.fin);
    mbar_wait_warp(sm.fin, 0, nullptr, 66);
    __syncwarp();
    bwd_teardown(true, tmem, Cfg::TMEM_COLS);
  } else if (warp >= 4) {
    // ---- P^T, dS^T for half c = (warp - 4) / 4: one key row per thread, 64 queries
    const int c = (warp - 4) >> 2, wl = warp & 3;
    const int kr = wl * 32 + lane, key = kt * 128 + kr;
    const uint32_t lane_addr = tmem + ((uint32_t)(wl * 32) << 16);
    const int shift = p.Sk - p.Sq;
    const f32x2 c2x2 = pack_f2(p.c2, p.c2);
    bool ok = true;
    for (int n = 0; n < nsteps; ++n) {
      ok = mbar_wait_warp(&sm.s_ready[c], n & 1, sm.abort_flag, 67 + c);
      // the step's lse2 / Delta rows: visible to this thread once it has seen their load
      // complete (the slot cannot be refilled before this warpgroup releases the step)
      if (ok) ok = mbar_wait_warp(&sm.full[n % Cfg::STAGES], (n / Cfg::STAGES) & 1, sm.abort_flag, 71);
      if (!ok) break;
      tc_fence_after();
      const float* vec = reinterpret_cast<const float*>(sm.slot(n % Cfg::STAGES) + 2 * Cfg::TILE);
      const int qbase = step_qt(n) * 128 + 64 * c;
      // visible queries of this key row: q >= key - shift (causal), q < Sq; none past Sk
      const int lo = p.causal ? key - shift - qbase : 0;
      const int hi = key < p.Sk ? min(64, p.Sq - qbase) : 0;
      const f32x2* nl2 = reinterpret_cast<const f32x2*>(vec + 64 * c);
      const f32x2* nd2 = reinterpret_cast<const f32x2*>(vec + 128 + 64 * c);
      bwd_half<BF16, true>(lane_addr + Cfg::S_COL + 64 * c, lane_addr + Cfg::DP_COL + 64 * c, c2x2,
                           [&](int j) { return nl2[j]; }, [&](int j) { return nd2[j]; }, lo, hi);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_ready[c]);
    }
    // ---- epilogue: warpgroup 0 writes dV, warpgroup 1 dK * scale (rows of real keys)
    if (ok) ok = mbar_wait_warp(sm.fin, 0, sm.abort_flag, 70);
    if (ok && !*sm.abort_flag) {
      tc_fence_after();
      void* out = c == 0 ? p.dv : p.dk;
      uint16_t* row = reinterpret_cast<uint16_t*>(out) + (((size_t)b * p.Sk + key) * p.Hkv + kvh) * D;
      bwd_store_row<BF16, D>(lane_addr + (c == 0 ? Cfg::ACC0 : Cfg::ACC1), c == 0 ? 1.f : p.scale, row,
                             key < p.Sk, nsteps == 0);
    }
    bwd_teardown(false, tmem, Cfg::TMEM_COLS);
  } else {
    bwd_teardown(false, tmem, Cfg::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- dQ
template <int D, bool BF16>
__global__ void __launch_bounds__(384, 1)
attn_bwd_q(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
           const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
           const BwdParams p) {
  using Cfg = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const BwdSmem<D> sm(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // one flat grid, longest first: Q tile major from the last (causal: it sees the most
  // keys), then batch, then query head
  const int per_tile = p.Hq * p.B;
  const int qt = p.n_qt - 1 - (int)blockIdx.x / per_tile;
  const int b = ((int)blockIdx.x % per_tile) / p.Hq, h = (int)blockIdx.x % p.Hq;
  const int kvh = h / p.G;
  int kend = p.Sk;                                   // keys any row of the tile sees
  if (p.causal) kend = min(p.Sk, min(qt * 128 + 127, p.Sq - 1) + p.Sk - p.Sq + 1);
  const int nsteps = kend > 0 ? (kend + 127) / 128 : 0;
  if (threadIdx.x == 0) bwd_init(sm);
  if (warp == 0) { tmem_alloc(sm.tmem_holder, Cfg::TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_holder;

  if (warp == 1) {
    // ---- loads: Q and dO once, then (K, V) per step
    if (lane == 0) {
      bool ok = true;
      int issued = 0;
      tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_do); tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_v);
      if (nsteps > 0) {
        mbar_arrive_expect_tx(sm.fix_full, 2 * Cfg::TILE);
        for (int c = 0; c < Cfg::KCH; ++c) {
          tma_load_4d(sm.fix0 + c * Cfg::CHUNK, &tm_q, sm.fix_full, c * 64, h, qt * 128, b);
          tma_load_4d(sm.fix1 + c * Cfg::CHUNK, &tm_do, sm.fix_full, c * 64, h, qt * 128, b);
        }
      }
      for (int n = 0; n < nsteps && ok; ++n) {
        const int s = n % Cfg::STAGES;
        if (n >= Cfg::STAGES) {
          ok = mbar_wait(&sm.empty[s], ((n / Cfg::STAGES) - 1) & 1, sm.abort_flag, 74);
          if (!ok) break;
        }
        uint8_t* dst = sm.slot(s);
        mbar_arrive_expect_tx(&sm.full[s], 2 * Cfg::TILE);
        for (int c = 0; c < Cfg::KCH; ++c) {
          tma_load_4d(dst + c * Cfg::CHUNK, &tm_k, &sm.full[s], c * 64, kvh, n * 128, b);
          tma_load_4d(dst + Cfg::TILE + c * Cfg::CHUNK, &tm_v, &sm.full[s], c * 64, kvh, n * 128, b);
        }
        issued = n + 1;
      }
      if (!ok) bwd_drain(sm, nsteps > 0, issued);
    }
    __syncwarp();
    bwd_teardown(false, tmem, Cfg::TMEM_COLS);
  } else if (warp == 0) {
    // ---- MMA issue
    constexpr uint32_t IDESC_S = idesc_f16(BF16 ? 1 : 0, 128, 64, 0, 0);
    constexpr uint32_t IDESC_ACC = idesc_f16(BF16 ? 1 : 0, 128, D, 0, 1);
    const uint32_t q_addr = smem_u32(sm.fix0), do_addr = smem_u32(sm.fix1);
    bool ok = nsteps == 0 || mbar_wait_warp(sm.fix_full, 0, sm.abort_flag, 75);
    if (ok) {
      // S half h = Q K[h]^T, dP half h = dO V[h]^T  (M = 128 queries, N = 64 keys)
      auto issue_s = [&](int n, int hh) {
        const uint32_t k_addr = smem_u32(sm.slot(n % Cfg::STAGES)), v_addr = k_addr + Cfg::TILE;
#pragma unroll
        for (int c = 0; c < Cfg::KCH; ++c)
          mma_ss_x4(tmem + Cfg::S_COL + 64 * hh, smem_desc_sw128(q_addr + c * Cfg::CHUNK, 16, 1024),
                    smem_desc_sw128(k_addr + c * Cfg::CHUNK + hh * 8192, 16, 1024), IDESC_S, c > 0);
#pragma unroll
        for (int c = 0; c < Cfg::KCH; ++c)
          mma_ss_x4(tmem + Cfg::DP_COL + 64 * hh, smem_desc_sw128(do_addr + c * Cfg::CHUNK, 16, 1024),
                    smem_desc_sw128(v_addr + c * Cfg::CHUNK + hh * 8192, 16, 1024), IDESC_S, c > 0);
        mma_commit_warp(&sm.s_ready[hh]);
      };
      // dQ += dS[h] K[h]  (K = the half's 64 keys; K read MN-major)
      auto issue_acc = [&](int n, int hh) {
        const uint32_t k_addr = smem_u32(sm.slot(n % Cfg::STAGES));
        mma_ts_x4(tmem + Cfg::ACC0, tmem + Cfg::DP_COL + 64 * hh,
                  smem_desc_sw128(k_addr + hh * 8192, Cfg::CHUNK, 1024), IDESC_ACC, (n > 0 || hh > 0) ? 1u : 0u);
      };
      ok = bwd_mma_loop<D>(sm, nsteps, issue_s, issue_acc);
    }
    if (!ok) *sm.abort_flag = 1;
    mma_commit_warp(sm.fin);
    mbar_wait_warp(sm.fin, 0, nullptr, 76);
    __syncwarp();
    bwd_teardown(true, tmem, Cfg::TMEM_COLS);
  } else if (warp >= 4) {
    // ---- dS for half c: one query row per thread, 64 keys
    const int c = (warp - 4) >> 2, wl = warp & 3;
    const int qr = wl * 32 + lane, q = qt * 128 + qr;
    const uint32_t lane_addr = tmem + ((uint32_t)(wl * 32) << 16);
    const size_t vrow = ((size_t)b * p.Hq + h) * p.sq_pad + q;     // q < sq_pad always
    const float nl1 = p.nlse2[vrow], nd1 = p.ndelta[vrow];
    const int klim = p.causal ? q + p.Sk - p.Sq : p.Sk - 1;          // last key this row sees
    const f32x2 c2x2 = pack_f2(p.c2, p.c2);
    const f32x2 nlp = pack_f2(nl1, nl1), ndp = pack_f2(nd1, nd1);
    bool ok = true;
    for (int n = 0; n < nsteps; ++n) {
      ok = mbar_wait_warp(&sm.s_ready[c], n & 1, sm.abort_flag, 77 + c);
      if (!ok) break;
      tc_fence_after();
      const int kbase = n * 128 + 64 * c;
      // visible keys of this row: k <= klim, k < Sk; none for padding rows
      const int hi = q < p.Sq ? min(p.Sk, klim + 1) - kbase : 0;
      bwd_half<BF16, false>(lane_addr + Cfg::S_COL + 64 * c, lane_addr + Cfg::DP_COL + 64 * c, c2x2,
                            [&](int) { return nlp; }, [&](int) { return ndp; }, 0, hi);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_ready[c]);
    }
    // ---- epilogue: warpgroup c writes dQ columns [c D/2, (c+1) D/2) * scale
    if (ok) ok = mbar_wait_warp(sm.fin, 0, sm.abort_flag, 80);
    if (ok && !*sm.abort_flag) {
      tc_fence_after();
      uint16_t* row = reinterpret_cast<uint16_t*>(p.dq) + (((size_t)b * p.Sq + q) * p.Hq + h) * D + c * (D / 2);
      bwd_store_row<BF16, D / 2>(lane_addr + Cfg::ACC0 + c * (D / 2), p.scale, row, q < p.Sq, nsteps == 0);
    }
    bwd_teardown(false, tmem, Cfg::TMEM_COLS);
  } else {
    bwd_teardown(false, tmem, Cfg::TMEM_COLS);
  }
}

}  // namespace sa
