// diag.cuh -- diagnostic kernels beside the attention path (never called by it).
//
//   * read_floor_ld / read_floor_bulk: read a buffer once and fold it into one word, the
//     first with 128-bit loads from every thread, the second with bulk asynchronous copies
//     into a shared-memory ring the way the decode's split kernel streams K/V.  They give
//     the time a cold read of the decode's bytes takes with no attention arithmetic, the
//     floor the decode is measured against;
//   * diag_exp2_poly: the forward's FMA-pipe 2^x (exp2_poly_pair) on caller-chosen
//     arguments, so its error can be checked on its own.
#pragma once
#include "ptx.cuh"
#include "fwd_sm100.cuh"

namespace sa {

// Block b reads 16-byte words [b n / G, (b + 1) n / G) of src, kUnroll independent loads per
// thread in flight, and XORs them into *sink (one atomic per warp).
constexpr int kFloorThreads = 256, kFloorUnroll = 8;

__global__ void __launch_bounds__(kFloorThreads)
read_floor_ld(const uint4* __restrict__ src, size_t n16, unsigned int* sink) {
  const size_t lo = n16 * blockIdx.x / gridDim.x, hi = n16 * (blockIdx.x + 1) / gridDim.x;
  uint32_t acc = 0;
  for (size_t base = lo; base < hi; base += (size_t)kFloorThreads * kFloorUnroll) {
    uint4 v[kFloorUnroll];
#pragma unroll
    for (int u = 0; u < kFloorUnroll; ++u) {
      const size_t i = base + (size_t)u * kFloorThreads + threadIdx.x;
      v[u] = i < hi ? __ldcs(src + i) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kFloorUnroll; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) atomicXor(sink, acc);
}

// Thread 0 of each block keeps kBulkStages bulk copies of up to kBulkBytes in flight over the
// block's contiguous range (16-byte aligned pieces); every thread XORs its share of each
// landed piece, and the slot is refilled once all have (the decode's split kernel consumes
// its K/V stages the same way).
constexpr int kBulkStages = 4, kBulkBytes = 16384;

__global__ void __launch_bounds__(128)
read_floor_bulk(const uint8_t* __restrict__ src, size_t n16, unsigned int* sink) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* ring = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(ring + kBulkStages * kBulkBytes);
  const size_t lo = 16 * (n16 * blockIdx.x / gridDim.x), hi = 16 * (n16 * (blockIdx.x + 1) / gridDim.x);
  const int npiece = (int)((hi - lo + kBulkBytes - 1) / kBulkBytes);
  auto piece_bytes = [&](int piece) -> uint32_t {
    const size_t off = lo + (size_t)piece * kBulkBytes;
    return (uint32_t)(hi - off < (size_t)kBulkBytes ? hi - off : (size_t)kBulkBytes);
  };
  auto issue = [&](int piece) {
    const int slot = piece % kBulkStages;
    mbar_arrive_expect_tx(&full[slot], piece_bytes(piece));
    bulk_copy_g2s(ring + slot * kBulkBytes, src + lo + (size_t)piece * kBulkBytes, piece_bytes(piece), &full[slot]);
  };
  if (threadIdx.x == 0) {
    for (int i = 0; i < kBulkStages; ++i) mbar_init(&full[i], 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    for (int i = 0; i < kBulkStages && i < npiece; ++i) issue(i);
  int issued = npiece < kBulkStages ? npiece : kBulkStages;
  uint32_t acc = 0;
  bool ok = true;
  for (int i = 0; i < npiece; ++i) {
    const int slot = i % kBulkStages;
    const bool landed = mbar_wait(&full[slot], (i / kBulkStages) & 1, nullptr, 60);
    const uint4* w = reinterpret_cast<const uint4*>(ring + slot * kBulkBytes);
    const int n = (int)(piece_bytes(i) / 16);
    for (int j = threadIdx.x; j < n; j += 128) {
      const uint4 x = w[j];
      acc ^= x.x ^ x.y ^ x.z ^ x.w;
    }
    if (!__syncthreads_and(landed)) { ok = false; break; }
    if (threadIdx.x == 0 && i + kBulkStages < npiece) issue(i + kBulkStages);
    if (i + kBulkStages < npiece) ++issued;
  }
  if (!ok && threadIdx.x == 0) {
    // every copy issued lands before shared memory goes away
    for (int i = issued > kBulkStages ? issued - kBulkStages : 0; i < issued; ++i)
      mbar_wait(&full[i % kBulkStages], (i / kBulkStages) & 1, nullptr, 61);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) atomicXor(sink, acc);
  __syncthreads();
}

// y[i] = 2^x[i] through the forward's FMA-pipe exponential, two arguments per thread.
__global__ void diag_exp2_poly(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x1 = i + 1 < n ? x[i + 1] : 0.f;
  float a, b;
  exp2_poly_pair(x[i], x1, a, b);
  y[i] = a;
  if (i + 1 < n) y[i + 1] = b;
}

}  // namespace sa
