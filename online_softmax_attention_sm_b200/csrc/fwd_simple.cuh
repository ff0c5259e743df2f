// fwd_simple.cuh -- plain CUDA-core attention forward (diagnostic cross-check only) and
// the fill kernel for the no-key case.
//
// One thread per query row runs the StreamAttention page's recurrence ("Kernel Design
// (Fused Online Softmax)") one key at a time in fp32: running max, running sum,
// rescaled accumulator, then acc / sum and lse = max + log(sum).
#pragma once
#include "ptx.cuh"
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <type_traits>

namespace sa {

template <bool BF16>
__device__ __forceinline__ float ld_f(const void* p, size_t i) {
  if (BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  return __half2float(reinterpret_cast<const __half*>(p)[i]);
}

template <bool BF16>
__device__ __forceinline__ void st_f(void* p, size_t i, float v) {
  if (BF16) reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else reinterpret_cast<__half*>(p)[i] = __float2half_rn(v);
}

template <int D, bool BF16>
__global__ void __launch_bounds__(64)
attn_fwd_simple(const void* q, const void* k, const void* v, void* o, float* lse,
                int Sq, int Sk, int Hq, int Hkv, int causal, float c2) {
  const int row = blockIdx.x * blockDim.x + threadIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  if (row >= Sq) return;
  const int kvh = h / (Hq / Hkv);
  float qr[D], acc[D];
  const size_t qoff = (((size_t)b * Sq + row) * Hq + h) * D;
#pragma unroll
  for (int d = 0; d < D; ++d) { qr[d] = ld_f<BF16>(q, qoff + d); acc[d] = 0.f; }
  int klim = Sk;
  if (causal) klim = max(0, min(Sk, row + Sk - Sq + 1));
  float m = -INFINITY, l = 0.f;
  for (int j = 0; j < klim; ++j) {
    const size_t koff = (((size_t)b * Sk + j) * Hkv + kvh) * D;
    float s = 0.f;
#pragma unroll
    for (int d = 0; d < D; ++d) s = fmaf(qr[d], ld_f<BF16>(k, koff + d), s);
    s *= c2;                                   // log2 domain
    const float mn = fmaxf(m, s);
    const float alpha = exp2f(m - mn);         // 0 on the first key (m = -inf)
    const float pj = exp2f(s - mn);
    l = l * alpha + pj;
#pragma unroll
    for (int d = 0; d < D; ++d) acc[d] = fmaf(pj, ld_f<BF16>(v, koff + d), acc[d] * alpha);
    m = mn;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int d = 0; d < D; ++d) st_f<BF16>(o, qoff + d, acc[d] * inv);
  if (lse) lse[((size_t)b * Hq + h) * Sq + row] = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
}

// No visible key at all (Sk == 0): O = 0, LSE = -inf.
__global__ void attn_fill_empty(uint16_t* o, size_t n_o, float* lse, size_t n_lse) {
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n_o; i += stride) o[i] = 0;
  if (lse)
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n_lse; i += stride) lse[i] = -INFINITY;
}

// Self-test of the bounded-wait path: one thread waits on an mbarrier that nothing ever
// completes.  The wait gives up after kWaitLimitNs, records a timeout in the status word
// and the kernel returns normally -- no trap, no fault, the context stays usable.
__global__ void selftest_bounded_wait() {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);          // expects one arrival that never comes
    abort_flag = 0;
    fence_barrier_init();
    mbar_wait(&bar, 0, &abort_flag, 99);
  }
}

}  // namespace sa
