// decode.cuh -- split-KV single-token decode and its LSE-weighted combine, sm_100a.
//
// Method: the StreamAttention page's split-state prototype ("Engine Direction": write
// partial online-softmax states, merge them in a second kernel) and its log-sum-exp
// weighted combining ("Distributed and Long-Context Variants").  Each split runs the
// online-softmax recurrence of "Kernel Design" over its slice of keys; the combine
// rescales every split's state to the common max and divides once.
//
// B200 design:
//   * grid (split, KV head x head-group, batch), about three CTAs per SM; the
//     G = Hq/Hkv query heads that share a KV head are packed as the rows of one 16-row
//     mma.sync tile, so every K/V byte is read from HBM exactly once (never once per
//     query head);
//   * thread 0 streams 64-token K and V slices with TMA tensor loads (128-byte swizzle)
//     into a ring of shared-memory stages; 4 warps each take 16 tokens of a stage;
//   * S = Q K^T and O += P V on mma.sync.m16n8k16 (fp32 accumulate), fragments from
//     ldmatrix; row max / sum by quad shuffles; the 4 warps merge through shared memory;
//   * paged K/V caches (the `PAGED` instance): a split looks up the cache page of each of
//     its 64-token stages in the block table once, and TMA reads (row in page, page)
//     instead of (token, batch); sequences have their own lengths;
//   * each split writes (unnormalised O, running max, two running sums) in fp32 to the
//     workspace; a combine kernel with one CTA per (batch, query head) merges them.  It
//     is launched with programmatic dependent launch, so its launch overlaps the split
//     grid (the page's two-kernel prototype lost to launch and merge overhead).
#pragma once
#include "ptx.cuh"
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <type_traits>

namespace sa {

template <int D>
struct DecCfg {
  static constexpr int TOK = 64;                       // tokens per stage
  static constexpr int KCH = D / 64;
  static constexpr int CHUNK_BYTES = TOK * 128;        // 64 tokens x 64 elements
  static constexpr int KV_BYTES = KCH * CHUNK_BYTES;   // one K (or V) stage
  static constexpr int STAGES = (D == 64) ? 4 : 2;
  static constexpr int SMEM_STAGES = STAGES * 2 * KV_BYTES;
  // write_partial's buffers; decode_merge uses the SMEM_STAGES region
  static constexpr int SMEM_MERGE = 4 * 16 * (D + 4) * 4 + 3 * 4 * 16 * 4;
  // paged K/V: the cache page of each stage of a split, looked up once at the start
  static constexpr int MAX_PAGED_STAGES = 256;         // a split covers at most 16384 tokens
  static constexpr int SMEM_TOTAL = 1024 + (SMEM_STAGES > SMEM_MERGE ? SMEM_STAGES : SMEM_MERGE) + 256 +
                                    MAX_PAGED_STAGES * 4;
};

// Workspace layout (caller-owned scratch, contents irrelevant between calls):
//   ws_ml [B, Hq, nsplit, 4] fp32 (max, 16-bit-weight sum, fp32 sum, pad),
//   then ws_o [B, Hq, nsplit, D] fp32.
struct DecParams {
  const void* q;       // [B, Hq, D]
  float* ws_o;         // [B, Hq, nsplit, D]
  float* ws_ml;        // [B, Hq, nsplit, 4]: max (log2 units of c2*s), 16-bit-weight sum, fp32 sum, 0
  void* o;             // [B, Hq, D]
  float* lse;          // [B, Hq] or null
  int B, Sk, Hq, Hkv, G, ngrp, nsplit, chunk;
  float c2;
  // paged K/V (attn_decode_split<.., PAGED = true>): caches [num_pages, page_size, Hkv, D];
  // the keys of sequence b are tokens 0 .. seqlens[b]-1, token t in page
  // block_table[b * max_blocks + t / page_size] at row t % page_size
  const int* block_table;   // [B, max_blocks]
  const int* seqlens;       // [B]
  int max_blocks, page_size;
  // single-kernel instance (attn_decode_split<.., FUSED = true>): one arrival counter per
  // (batch, KV head, head group) tile, zero at launch; the tile's last split merges and
  // zeroes it again
  unsigned int* sem;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

template <bool BF16>
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if (BF16) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if (BF16) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  } else {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
}

template <bool BF16>
__device__ __forceinline__ float unpack_sum(uint32_t v) {
  if (BF16) return __uint_as_float(v << 16) + __uint_as_float(v & 0xffff0000u);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&v));
  return f.x + f.y;
}

// Byte offset of (row, 16-byte column chunk) inside a 128-byte-swizzled box of 128-byte rows.
__device__ __forceinline__ uint32_t sw128(int row, int chunk16) {
  return (uint32_t)(row * 128 + ((chunk16 ^ (row & 7)) << 4));
}

// The 4 warps' states (each over its 16 tokens of every stage) are rescaled to the CTA
// max through shared memory and written as this split's partial state.
template <int D>
__device__ __forceinline__ void write_partial(const DecParams& p, uint8_t* smem, int b, int h0, int nrows,
                                              int split, int warp, int lane, const float (&o)[D / 8][4],
                                              float m0, float m1, float l0, float l1, float e0, float e1) {
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  e0 += __shfl_xor_sync(0xffffffffu, e0, 1);
  e0 += __shfl_xor_sync(0xffffffffu, e0, 2);
  e1 += __shfl_xor_sync(0xffffffffu, e1, 1);
  e1 += __shfl_xor_sync(0xffffffffu, e1, 2);
  constexpr int LD = D + 4;                                  // padded row: no bank conflicts
  float* sm_o = reinterpret_cast<float*>(smem);              // [4][16][LD] (stages are drained)
  float* sm_m = sm_o + 4 * 16 * LD;                          // [4][16]
  float* sm_l = sm_m + 64;                                   // [4][16]
  float* sm_e = sm_l + 64;                                   // [4][16]
  const int r0 = lane >> 2, r1 = r0 + 8;
  if ((lane & 3) == 0) {
    sm_m[warp * 16 + r0] = m0; sm_m[warp * 16 + r1] = m1;
    sm_l[warp * 16 + r0] = l0; sm_l[warp * 16 + r1] = l1;
    sm_e[warp * 16 + r0] = e0; sm_e[warp * 16 + r1] = e1;
  }
  __syncthreads();
  float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
  for (int w = 0; w < 4; ++w) { M0 = fmaxf(M0, sm_m[w * 16 + r0]); M1 = fmaxf(M1, sm_m[w * 16 + r1]); }
  const float w0 = (m0 == -INFINITY) ? 0.f : ex2(m0 - M0);
  const float w1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - M1);
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    const int c = n * 8 + (lane & 3) * 2;
    *reinterpret_cast<float2*>(&sm_o[(warp * 16 + r0) * LD + c]) = make_float2(o[n][0] * w0, o[n][1] * w0);
    *reinterpret_cast<float2*>(&sm_o[(warp * 16 + r1) * LD + c]) = make_float2(o[n][2] * w1, o[n][3] * w1);
  }
  __syncthreads();
  const size_t ws_row0 = ((size_t)b * p.Hq + h0) * p.nsplit + split;   // row r -> + r * nsplit
  for (int i = threadIdx.x; i < nrows * D; i += blockDim.x) {
    const int r = i / D, d = i % D;
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) acc += sm_o[(w * 16 + r) * LD + d];
    p.ws_o[(ws_row0 + (size_t)r * p.nsplit) * D + d] = acc;
  }
  if (threadIdx.x < nrows) {
    const int r = threadIdx.x;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sm_m[w * 16 + r]);
    float L = 0.f, E = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float mw = sm_m[w * 16 + r];
      const float sc = (mw == -INFINITY) ? 0.f : ex2(mw - M);
      L += sm_l[w * 16 + r] * sc;
      E += sm_e[w * 16 + r] * sc;
    }
    *reinterpret_cast<float4*>(p.ws_ml + (ws_row0 + (size_t)r * p.nsplit) * 4) = make_float4(M, L, E, 0.f);
  }
}

// Splits are capped so the combine's per-row weight table stays small.
template <int D>
struct DecMerge {
  static constexpr int MAX_SPLITS = (D == 64) ? 192 : 96;
};

template <int D, bool BF16>
__device__ __forceinline__ void decode_merge_row(const DecParams& p, size_t row, float* s_w, float (*s_red)[4],
                                                 float4* s_acc);

// FUSED (the single-kernel instance, for small batches where a second launch costs more
// than it saves): after writing its partial state, each CTA takes a ticket on its tile's
// arrival counter, and the tile's last split merges the tile's query heads itself.
template <int D, bool BF16, bool PAGED, bool FUSED = false>
__global__ void __launch_bounds__(128, 3)
attn_decode_split(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const DecParams p) {
  using Cfg = DecCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int region = Cfg::SMEM_STAGES > Cfg::SMEM_MERGE ? Cfg::SMEM_STAGES : Cfg::SMEM_MERGE;
  uint64_t* full = (uint64_t*)(smem + region);
  volatile int* abort_flag = (volatile int*)(full + Cfg::STAGES);
  int* s_page = (int*)(smem + region + 256);            // PAGED: cache page of each stage

  // let the combine grid launch now (it waits for this grid's results before reading)
  asm volatile("griddepcontrol.launch_dependents;");
  const int split = blockIdx.x;
  const int kvh = blockIdx.y / p.ngrp;
  const int grp = blockIdx.y % p.ngrp;
  const int b = blockIdx.z;
  const int h0 = kvh * p.G + grp * 16;                  // first query head of this tile
  const int nrows = min(16, p.G - grp * 16);            // valid rows of the tile
  // keys of this sequence: Sk, or (paged) its own length, clamped to what its block table holds
  const int seqlen = PAGED ? max(0, min(__ldg(p.seqlens + b), p.max_blocks * p.page_size)) : p.Sk;
  const int tok0 = split * p.chunk;
  const int tok1 = min(seqlen, tok0 + p.chunk);
  const int nstage = tok1 > tok0 ? (tok1 - tok0 + Cfg::TOK - 1) / Cfg::TOK : 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (PAGED) {
    // a 64-token stage never crosses a page (pages are multiples of 64 tokens, stages start
    // on multiples of 64); the host keeps nstage <= MAX_PAGED_STAGES
    const int* bt = p.block_table + (size_t)b * p.max_blocks;
    for (int i = threadIdx.x; i < nstage; i += blockDim.x) s_page[i] = __ldg(bt + (tok0 + i * Cfg::TOK) / p.page_size);
  }
  // TMA coordinates (token row, batch or page) of stage st
  auto stage_row = [&](int st) { const int t = tok0 + st * Cfg::TOK; return PAGED ? t % p.page_size : t; };
  auto stage_outer = [&](int st) { return PAGED ? s_page[st] : b; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < Cfg::STAGES; ++i) mbar_init(&full[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_v);
    for (int s = 0; s < Cfg::STAGES && s < nstage; ++s) {
      uint8_t* dk = smem + s * 2 * Cfg::KV_BYTES;
      mbar_arrive_expect_tx(&full[s], 2 * Cfg::KV_BYTES);
      for (int c = 0; c < Cfg::KCH; ++c) {
        tma_load_4d(dk + c * Cfg::CHUNK_BYTES, &tm_k, &full[s], c * 64, kvh, stage_row(s), stage_outer(s));
        tma_load_4d(dk + Cfg::KV_BYTES + c * Cfg::CHUNK_BYTES, &tm_v, &full[s], c * 64, kvh, stage_row(s), stage_outer(s));
      }
    }
  }

  // Q fragments (A operand, 16 rows = packed query heads, K = D), rows >= nrows are 0
  uint32_t qa[D / 16][4];
  {
    const uint16_t* q16 = reinterpret_cast<const uint16_t*>(p.q);
    const int r0 = lane >> 2, r1 = r0 + 8, cc = (lane & 3) * 2;
    const size_t base = ((size_t)b * p.Hq + h0) * D;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int d0 = kk * 16 + cc;
      auto ld = [&](int r, int d) -> uint32_t {
        return r < nrows ? *reinterpret_cast<const uint32_t*>(q16 + base + (size_t)r * D + d) : 0u;
      };
      qa[kk][0] = ld(r0, d0);
      qa[kk][1] = ld(r1, d0);
      qa[kk][2] = ld(r0, d0 + 8);
      qa[kk][3] = ld(r1, d0 + 8);
    }
  }

  float o[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  // l: sums of the 16-bit weights (normalise O); e: sums of the fp32 weights (LSE)
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f, e0 = 0.f, e1 = 0.f;
  const float c2 = p.c2;
  const uint32_t smem_addr = smem_u32(smem);
  bool ok = true;
  int issued = min(Cfg::STAGES, nstage);               // stages whose loads were issued

  for (int st = 0; st < nstage; ++st) {
    const int slot = st % Cfg::STAGES;
    // on a failed wait the stage's contents are stale but in bounds; the CTA-wide vote
    // after the compute decides whether to stop
    const bool landed = mbar_wait(&full[slot], (st / Cfg::STAGES) & 1, abort_flag, 40);
    const uint32_t kb = smem_addr + slot * 2 * Cfg::KV_BYTES;
    const uint32_t vb = kb + Cfg::KV_BYTES;
    const int wt = warp * 16;                          // this warp's first token in the stage
    // ---- S (16 heads x 16 tokens) = Q K^T
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      // matrices: (tok 0-7, d 0-7), (tok 0-7, d 8-15), (tok 8-15, d 0-7), (tok 8-15, d 8-15)
      const int mi = lane >> 3, rr = lane & 7;
      const int tok = wt + ((mi >> 1) << 3) + rr;
      const int dchunk = (kk & 3) * 2 + (mi & 1);      // 16-byte chunk within the 64-wide box
      uint32_t b0, b1, b2, b3;
      ldsm_x4(kb + (kk >> 2) * Cfg::CHUNK_BYTES + sw128(tok, dchunk), b0, b1, b2, b3);
      mma16816<BF16>(s[0], qa[kk], b0, b1);
      mma16816<BF16>(s[1], qa[kk], b2, b3);
    }
    // ---- scale, mask tokens outside [tok0, tok1), online softmax
    const int tbase = tok0 + st * Cfg::TOK + wt + (lane & 3) * 2;
    float x[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tk = tbase + n * 8 + (e & 1);
        x[n][e] = (tk < tok1) ? s[n][e] * c2 : -INFINITY;
      }
    float mx0 = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
    float mx1 = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float u0 = (mn0 == -INFINITY) ? 0.f : mn0, u1 = (mn1 == -INFINITY) ? 0.f : mn1;
    const float a0 = ex2(m0 - u0), a1 = ex2(m1 - u1);
    m0 = mn0; m1 = mn1;
    float pr[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      pr[n][0] = ex2(x[n][0] - u0); pr[n][1] = ex2(x[n][1] - u0);
      pr[n][2] = ex2(x[n][2] - u1); pr[n][3] = ex2(x[n][3] - u1);
    }
#pragma unroll
    for (int n = 0; n < D / 8; ++n) { o[n][0] *= a0; o[n][1] *= a0; o[n][2] *= a1; o[n][3] *= a1; }
    // P as the A operand (16 heads x 16 tokens); the row sums add the rounded weights
    // the MMA uses, so O / l stays an exact weighted average of V
    uint32_t pa[4];
    pa[0] = pack2<BF16>(pr[0][0], pr[0][1]);
    pa[1] = pack2<BF16>(pr[0][2], pr[0][3]);
    pa[2] = pack2<BF16>(pr[1][0], pr[1][1]);
    pa[3] = pack2<BF16>(pr[1][2], pr[1][3]);
    l0 = l0 * a0 + unpack_sum<BF16>(pa[0]) + unpack_sum<BF16>(pa[2]);
    l1 = l1 * a1 + unpack_sum<BF16>(pa[1]) + unpack_sum<BF16>(pa[3]);
    e0 = e0 * a0 + pr[0][0] + pr[0][1] + pr[1][0] + pr[1][1];
    e1 = e1 * a1 + pr[0][2] + pr[0][3] + pr[1][2] + pr[1][3];
    // ---- O (16 x D) += P V; V slice [16 tokens][D] via transposed ldmatrix
#pragma unroll
    for (int n = 0; n < D / 8; n += 2) {
      // matrices: (tok 0-7, d n*8..), (tok 8-15, d n*8..), (tok 0-7, d (n+1)*8..), (tok 8-15, d (n+1)*8..)
      const int mi = lane >> 3, rr = lane & 7;
      const int tok = wt + ((mi & 1) << 3) + rr;
      const int dcol = n + (mi >> 1);                  // 8-element column block 0..D/8-1
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(vb + (dcol >> 3) * Cfg::CHUNK_BYTES + sw128(tok, dcol & 7), b0, b1, b2, b3);
      mma16816<BF16>(o[n], pa, b0, b1);
      mma16816<BF16>(o[n + 1], pa, b2, b3);
    }
    // every warp is done with this slot, and every thread saw its data land
    if (!__syncthreads_and(landed)) { ok = false; break; }
    if (threadIdx.x == 0 && st + Cfg::STAGES < nstage) {
      const int ns = st + Cfg::STAGES;
      issued = ns + 1;
      uint8_t* dk = smem + slot * 2 * Cfg::KV_BYTES;
      mbar_arrive_expect_tx(&full[slot], 2 * Cfg::KV_BYTES);
      for (int c = 0; c < Cfg::KCH; ++c) {
        tma_load_4d(dk + c * Cfg::CHUNK_BYTES, &tm_k, &full[slot], c * 64, kvh, stage_row(ns), stage_outer(ns));
        tma_load_4d(dk + Cfg::KV_BYTES + c * Cfg::CHUNK_BYTES, &tm_v, &full[slot], c * 64, kvh, stage_row(ns), stage_outer(ns));
      }
    }
  }
  if (!ok) {
    // drain loads still in flight before shared memory is released
    if (threadIdx.x == 0) {
      // loads were issued for stages 0 .. issued-1; those not yet consumed may be pending
      // (each slot's most recent load is among the last STAGES issued)
      for (int st = max(0, issued - Cfg::STAGES); st < issued; ++st)
        mbar_wait(&full[st % Cfg::STAGES], (st / Cfg::STAGES) & 1, nullptr, 41);
    }
    __syncthreads();
    return;                                                   // outputs undefined; status word set
  }
  write_partial<D>(p, smem, b, h0, nrows, split, warp, lane, o, m0, m1, l0, l1, e0, e1);
  if (FUSED) {
    // every thread's partial-state stores are visible device-wide before the ticket
    __threadfence();
    __syncthreads();
    volatile int* s_last = reinterpret_cast<volatile int*>(smem + region + 128);
    const unsigned tile = ((unsigned)b * gridDim.y + blockIdx.y);
    if (threadIdx.x == 0) *s_last = atomicAdd(p.sem + tile, 1u) == (unsigned)p.nsplit - 1u;
    __syncthreads();
    if (*s_last) {
      __threadfence();
      float* s_w = reinterpret_cast<float*>(smem);            // stages are drained
      float (*s_red)[4] = reinterpret_cast<float (*)[4]>(s_w + DecMerge<D>::MAX_SPLITS);
      float4* s_acc = reinterpret_cast<float4*>(s_w + DecMerge<D>::MAX_SPLITS + 16);
      for (int r = 0; r < nrows; ++r) decode_merge_row<D, BF16>(p, (size_t)b * p.Hq + h0 + r, s_w, s_red, s_acc);
      if (threadIdx.x == 0) p.sem[tile] = 0u;                  // ready for the next launch
    }
  }
}

// The merge's summation order, written out so the combine kernel and the single-kernel
// instance (which run the same row merge) give identical bits whatever the compiler does
// around them.
// With the split weights w_s = 2^(m_s - M), M the row max over the splits:
//   * each of the two sums (of the 16-bit weights, of the fp32 weights), sum_s w_s y_s:
//     virtual lane t of 128 (warp t / 32, lane t % 32) takes splits t and t + 128,
//     x_t = fma(w_b, y_b, w_a * y_a); a butterfly over the 32 lanes of each virtual warp;
//     then (x_0 + x_1) + (x_2 + x_3) over the 4 virtual warps;
//   * each output float4 column c: group g of NG = 128 / (D/4) sums its splits g, g + NG, ...
//     in order with fma from 0; then the NG group sums in order g = 0, 1, ...
// Every operation is written with an explicit rounding so no contraction differs between
// the two kernels.
__device__ __forceinline__ float merge_pair(float wa, float ya, float wb, float yb) {
  return __fmaf_rn(wb, yb, __fmul_rn(wa, ya));
}
__device__ __forceinline__ float butterfly_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = __fadd_rn(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;                                                   // the same value in every lane
}
__device__ __forceinline__ float sum4(const float (&x)[4]) {
  return __fadd_rn(__fadd_rn(x[0], x[1]), __fadd_rn(x[2], x[3]));
}
__device__ __forceinline__ void fma4(float4& acc, float w, const float4& v) {
  acc.x = __fmaf_rn(w, v.x, acc.x); acc.y = __fmaf_rn(w, v.y, acc.y);
  acc.z = __fmaf_rn(w, v.z, acc.z); acc.w = __fmaf_rn(w, v.w, acc.w);
}
__device__ __forceinline__ void add4(float4& a, const float4& b) {
  a.x = __fadd_rn(a.x, b.x); a.y = __fadd_rn(a.y, b.y); a.z = __fadd_rn(a.z, b.z); a.w = __fadd_rn(a.w, b.w);
}
template <bool BF16>
__device__ __forceinline__ void store_o4(const DecParams& p, size_t row, int D, int c, const float4& a, float L) {
  const float inv = L > 0.f ? 1.f / L : 0.f;
  uint2 packed;
  packed.x = pack2<BF16>(__fmul_rn(a.x, inv), __fmul_rn(a.y, inv));
  packed.y = pack2<BF16>(__fmul_rn(a.z, inv), __fmul_rn(a.w, inv));
  reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(p.o) + row * D)[c] = packed;
}
__device__ __forceinline__ float merged_lse(float M, float E) {
  return E > 0.f ? __fmul_rn(__fadd_rn(M, __log2f(E)), 0.69314718055994531f) : -INFINITY;
}

// The merge of one (batch, query head) row by a block of 128 threads (scratch: s_w [MAX_SPLITS],
// s_red [3][4], s_acc [128]).  Loads bypass L1 (.cg): in the single-kernel instance the
// partial states were written by other CTAs of the same grid.  Thread t owns float4 column
// c = t % (D/4) and the splits g, g + NG, ... with g = t / (D/4).
template <int D, bool BF16>
__device__ __forceinline__ void decode_merge_row(const DecParams& p, size_t row, float* s_w, float (*s_red)[4],
                                                 float4* s_acc) {
  constexpr int NC = D / 4, NG = 128 / NC;
  constexpr int MAXS = DecMerge<D>::MAX_SPLITS;
  constexpr int PER = (MAXS + NG - 1) / NG;                   // splits per thread, at most
  static_assert(MAXS <= 256, "two split maxima per thread");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ns = p.nsplit;
  const float4* ml = reinterpret_cast<const float4*>(p.ws_ml) + row * ns;
  const float4* os = reinterpret_cast<const float4*>(p.ws_o) + row * ns * NC;
  const int c = tid % NC, g = tid / NC;
  // all loads first
  const float4 ninf = make_float4(-INFINITY, 0.f, 0.f, 0.f);
  const float4 mlA = tid < ns ? __ldcg(ml + tid) : ninf;
  const float4 mlB = tid + 128 < ns ? __ldcg(ml + tid + 128) : ninf;
  float4 v[PER];
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int s = g + u * NG;
    v[u] = s < ns ? __ldcg(os + (size_t)s * NC + c) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // max over splits
  float M = fmaxf(mlA.x, mlB.x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) s_red[0][warp] = M;
  __syncthreads();
  M = fmaxf(fmaxf(s_red[0][0], s_red[0][1]), fmaxf(s_red[0][2], s_red[0][3]));
  // weights and the two sums
  const float wA = (mlA.x == -INFINITY) ? 0.f : ex2(mlA.x - M);
  const float wB = (mlB.x == -INFINITY) ? 0.f : ex2(mlB.x - M);
  if (tid < ns) s_w[tid] = wA;
  if (tid + 128 < ns) s_w[tid + 128] = wB;
  const float L = butterfly_sum(merge_pair(wA, mlA.y, wB, mlB.y));
  const float E = butterfly_sum(merge_pair(wA, mlA.z, wB, mlB.z));
  __syncthreads();                                            // s_red[0] consumed, s_w written
  if (lane == 0) { s_red[1][warp] = L; s_red[2][warp] = E; }
  // weighted sum of this thread's splits
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int s = g + u * NG;
    if (s < ns) fma4(acc, s_w[s], v[u]);
  }
  s_acc[tid] = acc;
  __syncthreads();
  const float Lt = sum4(s_red[1]), Et = sum4(s_red[2]);
  if (tid < NC) {
    float4 a = s_acc[tid];
#pragma unroll
    for (int k = 1; k < NG; ++k) add4(a, s_acc[k * NC + tid]);
    store_o4<BF16>(p, row, D, tid, a, Lt);
  }
  if (p.lse && tid == 0) p.lse[row] = merged_lse(M, Et);
  __syncthreads();                                            // scratch free for the next row
}

// Merge of every split's partial state for one (batch, query head) row per CTA:
//   M = max_s m_s,  w_s = 2^(m_s - M),  O = sum_s w_s O_s / sum_s w_s l_s,
//   LSE = (M + log2 sum_s w_s e_s) * ln 2.
// Launched with programmatic dependent launch right behind the split kernel: its CTAs are
// resident before the split grid ends and proceed the moment its results are visible.
// Every load (the split maxima/sums and the partial output rows) is issued up front, so
// the merge costs one round trip to L2.  Thread t owns float4 column c = t % (D/4) and the
// splits s = g, g + NG, ... with g = t / (D/4), NG = 128 / (D/4); the NG partial sums per
// column are added through shared memory.
template <int D, bool BF16>
__global__ void __launch_bounds__(128)
attn_decode_combine(const DecParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ float s_w[DecMerge<D>::MAX_SPLITS];
  __shared__ float s_red[3][4];
  __shared__ float4 s_acc[128];
  decode_merge_row<D, BF16>(p, blockIdx.x, s_w, s_red, s_acc);
}

}  // namespace sa
