// Block-sparse forward, first kernel: the per-unit K/V tile lists that the forward kernel's
// block-sparse instance (fwd_sm100.cuh, record layout at kSparseSlotBytes) walks.
#pragma once
#include "fwd_sm100.cuh"

namespace sa {

// Block-sparse forward: one warp per unit record (batch, head, 256-row query block).  A key
// tile is kept for a Q tile when the caller's block mask [B, Hq, ceil(Sq/128), ceil(Sk/128)]
// is nonzero there and the tile is not wholly past the causal diagonal.  The unit's list
// holds first the tiles both Q tiles keep (one load, both softmax warpgroups busy), then the
// tiles only one of them keeps, alternating between the two so that the warpgroups take
// turns (a run of one tile's steps would leave the other idle); ascending within each kind.
// The order of a Q tile's key tiles does not change its result beyond rounding.
__global__ void sparse_unit_lists(const uint8_t* __restrict__ mask, uint16_t* __restrict__ out, int B,
                                  int Hq, int Sq, int Sk, int causal, int n_qblk, int stride) {
  const int nq = (Sq + 127) / 128, nk = (Sk + 127) / 128;
  const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= (long long)B * Hq * n_qblk) return;
  const int qb = (int)(w % n_qblk);
  const long long bh = w / n_qblk;
  uint16_t* rec = out + (size_t)w * stride;
  const uint8_t* row[2];
  int kmax[2];
  for (int t = 0; t < 2; ++t) {
    const int r = 2 * qb + t;
    row[t] = nullptr;
    kmax[t] = -1;
    if (r < nq) {
      row[t] = mask + ((size_t)bh * nq + r) * nk;
      const int last = min(Sq, (r + 1) * 128) - 1 + Sk - Sq;   // last key the tile's last row sees
      kmax[t] = !causal ? nk - 1 : (last < 0 ? -1 : min(nk - 1, last / 128));
    }
  }
  auto keep = [&](int t, int kt) { return kt <= kmax[t] && row[t][kt] != 0; };
  // pass 1: counts (both, tile 0 in all, tile 1 in all)
  int nb = 0, n0 = 0, n1 = 0;
  for (int base = 0; base < nk; base += 32) {
    const int kt = base + lane;
    const unsigned b0 = __ballot_sync(~0u, keep(0, kt)), b1 = __ballot_sync(~0u, keep(1, kt));
    nb += __popc(b0 & b1);
    n0 += __popc(b0);
    n1 += __popc(b1);
  }
  const int m = min(n0 - nb, n1 - nb);    // single-tile entries that alternate
  // pass 2: each entry's position
  const unsigned lt = (1u << lane) - 1u;
  int cb = 0, c0 = 0, c1 = 0;
  for (int base = 0; base < nk; base += 32) {
    const int kt = base + lane;
    const bool k0 = keep(0, kt), k1 = keep(1, kt);
    const unsigned b0 = __ballot_sync(~0u, k0), b1 = __ballot_sync(~0u, k1);
    const unsigned bb = b0 & b1, s0 = b0 & ~b1, s1 = b1 & ~b0;
    int pos = -1;
    if (k0 && k1) {
      pos = cb + __popc(bb & lt);
    } else if (k0) {
      const int r = c0 + __popc(s0 & lt);
      pos = nb + (r < m ? 2 * r : 2 * m + (r - m));
    } else if (k1) {
      const int r = c1 + __popc(s1 & lt);
      pos = nb + (r < m ? 2 * r + 1 : 2 * m + (r - m));
    }
    if (pos >= 0) rec[8 + pos] = (uint16_t)(kt | ((int)k0 << 14) | ((int)k1 << 15));
    cb += __popc(bb);
    c0 += __popc(s0);
    c1 += __popc(s1);
  }
  const int nu = n0 + n1 - nb;
  if (lane < 8) rec[lane] = (uint16_t)(lane == 0 ? nu : lane == 1 ? n0 : lane == 2 ? n1 : 0);
}

}  // namespace sa
