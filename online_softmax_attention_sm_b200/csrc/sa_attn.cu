// sa_attn.cu -- host side of the C ABI declared in include/sa_attn.h: argument checks,
// tensor-map construction, split planning and kernel launches.  Nothing here allocates
// device memory; every device pointer belongs to the caller.
#include "../../include/sa_attn.h"
#include "ptx.cuh"
#include "fwd_sm100.cuh"
#include "fwd_pair_sm100.cuh"
#include "sparse_lists.cuh"
#include "bwd_sm100.cuh"
#include "fwd_simple.cuh"
#include "decode.cuh"
#include "diag.cuh"

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <tuple>
#include <mutex>
#include <atomic>
#include <vector>
#include <algorithm>
#include <string>

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(SA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// ---------------------------------------------------------------- tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Device address of a __device__ variable of this library on the current device, looked up
// once per (device, context, variable) with that device current and cached.  Keyed by the
// context too: after a device reset the runtime creates a new primary context and reloads
// the module, and the old address would be stale.  The context is identified by its
// process-unique id (cuCtxGetId), not its handle, which a new context could reuse.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

int device_symbol(const void* symbol, const char* what, void** out) {
  static std::mutex mu;
  static std::map<std::tuple<int, unsigned long long, uintptr_t>, void*> cache;
  static CtxGetCurrentFn ctx_fn = nullptr;
  static CtxGetIdFn id_fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      ctx_fn = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      id_fn = reinterpret_cast<CtxGetIdFn>(p);
  });
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  CUcontext ctx = nullptr;
  if (ctx_fn && (ctx_fn(&ctx) != CUDA_SUCCESS || !ctx)) {
    // no context current yet: the runtime makes the device's primary context current on
    // first use, which a no-op free triggers
    cudaFree(nullptr);
    if (ctx_fn(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  }
  unsigned long long ctx_key = reinterpret_cast<uintptr_t>(ctx);
  unsigned long long id = 0;
  if (ctx && id_fn && id_fn(ctx, &id) == CUDA_SUCCESS) ctx_key = id;
  const auto key = std::make_tuple(dev, ctx_key, reinterpret_cast<uintptr_t>(symbol));
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) { *out = it->second; return SA_OK; }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, symbol);
  if (e != cudaSuccess) return fail(SA_ERR_CUDA, "cudaGetSymbolAddress(%s): %s", what, cudaGetErrorString(e));
  if (cache.size() < 4096) cache[key] = p;
  *out = p;
  return SA_OK;
}

// Map element type for 8-bit (e4m3) tensors, next to SA_FP16 / SA_BF16.
constexpr int kMapU8 = 100;

// View a [B, S, H, D] 16-bit (or 8-bit) tensor as 4-D (D, H, S, B); box = one 128-byte row
// of elements (64, or 128 for 8-bit) x 1 head x `rows` rows x 1 batch, 128-byte swizzle.
// Rows past S read as zero.
int make_map(CUtensorMap* m, const void* ptr, int dtype, int D, int H, int S, int B, int rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t eb = dtype == kMapU8 ? 1 : 2;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * eb, (cuuint64_t)H * D * eb, (cuuint64_t)S * H * D * eb};
  cuuint32_t box[4] = {(cuuint32_t)(128 / eb), 1, (cuuint32_t)rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType ty = dtype == kMapU8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : dtype == SA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUresult r = enc(m, ty, 4, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return SA_OK;
}

// ---------------------------------------------------------------- device facts
int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

constexpr float kLog2e = 1.4426950408889634f;

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Shared checks of the shape arguments.  Returns SA_OK or an error code.
int check_dims(int B, int Sq, int Sk, int Hq, int Hkv, int D, int dtype, float scale) {
  if (B < 0 || Sq < 0 || Sk < 0 || Hq < 0 || Hkv < 0)
    return fail(SA_ERR_INVALID, "negative size (B=%d Sq=%d Sk=%d Hq=%d Hkv=%d)", B, Sq, Sk, Hq, Hkv);
  if (Hq > 0 && (Hkv == 0 || Hq % Hkv != 0))
    return fail(SA_ERR_INVALID, "Hq (%d) must be a positive multiple of Hkv (%d)", Hq, Hkv);
  if (D != 64 && D != 128) return fail(SA_ERR_UNSUPPORTED, "head dim D=%d not supported (64 or 128)", D);
  if (dtype != SA_FP16 && dtype != SA_BF16) return fail(SA_ERR_UNSUPPORTED, "unknown dtype %d", dtype);
  if (!std::isfinite(scale)) return fail(SA_ERR_INVALID, "scale must be finite");
  return SA_OK;
}

int check_ptrs(const void* q, const void* k, const void* v, const void* o, const void* lse) {
  if (!q || !k || !v || !o) return fail(SA_ERR_INVALID, "q, k, v and o must be non-null");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse && !aligned16(lse)))
    return fail(SA_ERR_INVALID, "tensor pointers must be 16-byte aligned");
  return SA_OK;
}

int launch_fill(void* o, size_t n_o, float* lse, size_t n_lse, cudaStream_t st) {
  size_t n = n_o > n_lse ? n_o : n_lse;
  int blocks = (int)((n + 255) / 256);
  if (blocks > 4 * num_sms()) blocks = 4 * num_sms();
  if (blocks < 1) blocks = 1;
  sa::attn_fill_empty<<<blocks, 256, 0, st>>>((uint16_t*)o, n_o, lse, n_lse);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "fill launch");
}

// Static-order imbalance of the forward kernel's unit list over ncta CTAs: the snake order
// (fwd_unit_of) with each unit costing its K/V tiles plus two tiles of per-unit overhead,
// max over CTAs / mean.  Mirrors fwd_unit (query block of a unit) and fwd_kv_tiles.
double static_imbalance(const sa::FwdParams& p, int ncta) {
  const int G = p.Hq / p.Hkv, n_bk = p.B * p.Hkv;
  auto tiles = [&](int r0) -> int {
    if (r0 >= p.Sq) return 0;
    int kend = p.Sk;
    if (p.causal) {
      const int rmax = std::min(r0 + 127, p.Sq - 1);
      kend = std::min(p.Sk, rmax + p.Sk - p.Sq + 1);
    }
    return kend > 0 ? (kend + 127) / 128 : 0;
  };
  std::vector<double> load(ncta, 0.0);
  const long long per_band = (long long)p.band * p.B * p.Hq;
  for (int u = 0; u < p.n_units; ++u) {
    const long long bi = u / per_band;
    const int bs = std::min<long long>(p.band, p.n_qblk - bi * p.band);
    const long long r = u - bi * per_band;
    const long long full_grp = (long long)p.kv_group * G * bs;
    const long long g = r / full_grp;
    const int gsize = (int)std::min<long long>(p.kv_group, n_bk - g * p.kv_group);
    const long long rr = r - g * full_grp;
    const int qb = p.n_qblk - 1 - (int)(bi * p.band + rr / ((long long)gsize * G));
    const int cost = std::max(tiles(qb * 256), tiles(qb * 256 + 128)) + 2;
    const int round = u / ncta, c = u % ncta;
    load[(round & 1) ? ncta - 1 - c : c] += cost;
  }
  double mx = 0, sum = 0;
  for (double l : load) { mx = std::max(mx, l); sum += l; }
  return sum > 0 ? mx * ncta / sum : 1.0;
}

// Whether the forward kernel should take its units dynamically, decided once per shape.
bool fwd_use_dynamic(const sa::FwdParams& p, int D, int ncta) {
  static std::mutex mu;
  static std::map<std::vector<long long>, bool> memo;
  const std::vector<long long> key = {p.B, p.Sq, p.Sk, p.Hq, p.Hkv, D, p.causal, ncta};
  std::lock_guard<std::mutex> lock(mu);
  auto it = memo.find(key);
  if (it != memo.end()) return it->second;
  // many rounds balance on their own; counting them would only cost host time
  const bool dyn = p.n_units <= 64 * ncta && static_imbalance(p, ncta) > 1.05;
  if (memo.size() < 4096) memo[key] = dyn;
  return dyn;
}

// Dynamic-scheduling counters of the forward kernel: kFwdWorkSlots pairs (next unit, CTAs
// done), zero-initialised with the module; launches of the dynamic instance take slots in
// turn and the last CTA of a launch zeroes its pair, so up to kFwdWorkSlots of them may be in
// flight at once (on any streams) without sharing a counter.  A launch that shared a pair
// with a live one would skip or repeat units; the limit is stated in the C ABI's header.
constexpr int kFwdWorkSlots = 1024;
static __device__ unsigned int g_fwd_work[2 * kFwdWorkSlots];

int fwd_work_slot(unsigned int** out) {
  static std::atomic<unsigned int> next{0};
  void* base = nullptr;
  int rc = device_symbol((const void*)&g_fwd_work, "forward work counters", &base);
  if (rc != SA_OK) return rc;
  *out = static_cast<unsigned int*>(base) + 2 * (next++ % kFwdWorkSlots);
  return SA_OK;
}

// Scheduling groups of the forward's unit order for ncta CTAs (or CTA pairs): (batch, KV
// head) pairs whose K + V (seq_k keys, row_bytes per key of each) fit in half the L2; among
// the admissible sizes the one whose band (ceil(ncta / (kv_group * G)) query blocks) fills
// whole rounds most exactly, then the smaller.
void plan_units(sa::FwdParams& p, int ncta, int seq_k, double row_bytes) {
  int dev = 0, l2 = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess)
    l2 = 64 << 20;
  const int G = p.Hq / p.Hkv, n_bk = p.B * p.Hkv;
  const double kv_bytes = 2.0 * seq_k * row_bytes;   // K and V of one (b, KV head)
  long long gmax = (long long)((l2 / 2) / kv_bytes);
  if (gmax < 1) gmax = 1;
  if (gmax > n_bk) gmax = n_bk;
  int best_g = 1, best_band = 1;
  double best_waste = 1e30;
  for (int g = 1; g <= gmax; ++g) {
    const int band = (ncta + g * G - 1) / (g * G);
    const double waste = (double)((long long)band * g * G % ncta) / ncta;   // partial round
    if (waste < best_waste - 1e-9) { best_waste = waste; best_g = g; best_band = band; }
  }
  p.kv_group = best_g;
  p.band = best_band;
  if (best_band >= p.n_qblk && p.n_qblk > 4) {
    // short sequences: one band would hold every query block, so a round would mix the
    // longest and shortest units of a few pairs; take the units longest first across
    // all pairs instead (bands of one query block, one group).  Measured: 3-26 % faster
    // for sequences of 2048-8192 tokens and packed mixes; at 1024 tokens (4 query
    // blocks) the pair-by-pair order was 4 % faster and stays
    p.band = 1;
    p.kv_group = n_bk;
  } else if (p.band > p.n_qblk) {
    p.band = p.n_qblk;
  }
}

// The dense 16-bit forward at D = 128 on CTA pairs (attn_fwd_pair_sm100): p holds the
// problem (dense layout, static order); the grid is as many clusters of two as fit at once
// (at most one per two SMs), the unit order planned for that many.
template <bool BF16>
int launch_fwd_pair(const void* q, const void* k, const void* v, sa::FwdParams p, int seq_k, cudaStream_t st) {
  using Cfg = sa::PairCfg;
  const int ty = BF16 ? SA_BF16 : SA_FP16;
  CUtensorMap mq, mk, mv;
  int rc;
  if ((rc = make_map(&mq, q, ty, 128, p.Hq, p.Sq, p.B, 128)) != SA_OK) return rc;
  if ((rc = make_map(&mk, k, ty, 128, p.Hkv, p.Sk, p.B, 64)) != SA_OK) return rc;     // 64-key halves
  if ((rc = make_map(&mv, v, ty, 128, p.Hkv, p.Sk, p.B, 128)) != SA_OK) return rc;
  auto kern = sa::attn_fwd_pair_sm100<BF16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_TOTAL);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attn_fwd_pair_sm100)");
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(Cfg::THREADS);
  cfg.dynamicSmemBytes = Cfg::SMEM_TOTAL;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static int max_cl[64] = {0};
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(SA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  if (!max_cl[dev]) {
    cfg.gridDim = dim3(2 * (num_sms() / 2));
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveClusters(attn_fwd_pair_sm100)");
    if (n <= 0) return fail(SA_ERR_UNSUPPORTED, "no CTA pair of the forward fits on this device");
    max_cl[dev] = n < num_sms() / 2 ? n : num_sms() / 2;
  }
  const int ncl = p.n_units < max_cl[dev] ? p.n_units : max_cl[dev];
  plan_units(p, ncl, seq_k, 256.0);
  cfg.gridDim = dim3(2 * ncl);
  e = cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, p);
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "attn_fwd_pair_sm100 launch");
}

// Packed variable-length sequences for launch_fwd (cu_q null: the dense layout).
struct FwdVarlen {
  const int* cu_q = nullptr;
  const int* cu_k = nullptr;
  int max_sq = 0, max_sk = 0;
  // paged K/V (block_table set): caches [num_pages, page_size, Hkv, D], key lengths seqlens_k
  const int* block_table = nullptr;
  const int* seqlens_k = nullptr;
  int max_blocks = 0, page_size = 0, num_pages = 0;
};

// Block-sparse unit records for launch_fwd (sp null: every key tile up to the diagonal).
struct FwdSparse {
  const uint16_t* sp = nullptr;
  int stride = 0;   // uint16 per record
};

// uint16 per block-sparse unit record for Sk keys: 8 header slots + the longest list,
// rounded up to 16 bytes.
int sparse_stride(int Sk) { return 8 + (((Sk + 127) / 128 + 7) / 8) * 8; }

// Dense: q/o [B, Sq, Hq, D], k/v [B, Sk, Hkv, D].  Packed (vl.cu_q set): B sequences,
// q/o [Sq, Hq, D] and k/v [Sk, Hkv, D] with Sq, Sk the totals, LSE [Hq, Sq].
// Block-sparse (sparse.sp set, dense layout): the unit records built by sparse_unit_lists.
// FP8: q, k, v are e4m3, o bf16; `scale` already holds the Q and K descales, o_mul the V
// descale.
template <int D, bool BF16, bool FP8 = false>
int launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Sq,
               int Sk, int Hq, int Hkv, int causal, float scale, cudaStream_t st,
               const FwdVarlen& vl = FwdVarlen(), const FwdSparse& sparse = FwdSparse(), float o_mul = 1.f,
               bool force_pair = false) {
  using Cfg = sa::FwdCfg<D, FP8>;
  const bool packed = vl.cu_q != nullptr;
  const int map_b = packed ? 1 : B;
  const int map_ty = FP8 ? kMapU8 : (BF16 ? SA_BF16 : SA_FP16);
  CUtensorMap mq, mk, mv;
  int rc;
  if ((rc = make_map(&mq, q, map_ty, D, Hq, Sq, map_b, 128)) != SA_OK) return rc;
  const bool paged = vl.block_table != nullptr;
  const int k_rows = paged ? vl.page_size : Sk, k_outer = paged ? vl.num_pages : map_b;
  if ((rc = make_map(&mk, k, map_ty, D, Hkv, k_rows, k_outer, 128)) != SA_OK) return rc;
  if ((rc = make_map(&mv, v, map_ty, D, Hkv, k_rows, k_outer, 128)) != SA_OK) return rc;
  sa::FwdParams p;
  p.o = o; p.lse = lse;
  p.B = B; p.Sq = Sq; p.Sk = Sk; p.Hq = Hq; p.Hkv = Hkv; p.causal = causal;
  p.cu_q = vl.cu_q; p.cu_k = vl.cu_k;
  p.block_table = vl.block_table; p.seqlens_k = vl.seqlens_k;
  p.max_blocks = vl.max_blocks; p.page_size = vl.page_size;
  p.max_sq = packed ? vl.max_sq : Sq;
  p.sp = sparse.sp; p.sp_stride = sparse.stride;
  p.o_mul = o_mul;
  const int seq_k = packed ? (vl.max_sk > 0 ? vl.max_sk : 1) : Sk;   // one sequence's keys, for L2 grouping
  p.n_qblk = (p.max_sq + 255) / 256;
  long long units = (long long)B * Hq * p.n_qblk;
  if (units > 0x7fffffffLL) return fail(SA_ERR_UNSUPPORTED, "too many work units (%lld)", units);
  p.n_units = (int)units;
  p.c2 = scale * kLog2e;
  if ((rc = fwd_work_slot(&p.work)) != SA_OK) return rc;
  plan_units(p, p.n_units < num_sms() ? p.n_units : num_sms(), seq_k, (double)D * (FP8 ? 1 : 2));
  const int grid = p.n_units < num_sms() ? p.n_units : num_sms();
  // the CTA-pair kernel when asked for (sa_attn_fwd_pair; dense 16-bit, D = 128): measured
  // slower than this kernel on every shape tried, so sa_attn_fwd does not take it
  if constexpr (!FP8 && D == 128) {
    if (force_pair && !packed && !paged && !sparse.sp) return launch_fwd_pair<BF16>(q, k, v, p, seq_k, st);
  }
  // packed lengths and block-sparse lists live on the device, so the static order's
  // balance is unknown: dynamic
  decltype(&sa::attn_fwd_sm100<D, BF16, false, false, FP8>) kern;
  if constexpr (FP8) {
    kern = sparse.sp ? sa::attn_fwd_sm100<D, BF16, true, true, true>
         : (packed || fwd_use_dynamic(p, D, grid)) ? sa::attn_fwd_sm100<D, BF16, true, false, true>
                                                   : sa::attn_fwd_sm100<D, BF16, false, false, true>;
  } else {
    kern = sparse.sp ? sa::attn_fwd_sm100<D, BF16, true, true>
         : paged ? sa::attn_fwd_sm100<D, BF16, true, false, false, true>
         : (packed || fwd_use_dynamic(p, D, grid)) ? sa::attn_fwd_sm100<D, BF16, true, false>
                                                   : sa::attn_fwd_sm100<D, BF16, false, false>;
  }
  const int smem = Cfg::SMEM_TOTAL + (sparse.sp ? Cfg::SMEM_SPARSE : 0);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attn_fwd_sm100)");
  // the in-kernel register reallocation must fit in what the block is launched with,
  // otherwise the increasing warpgroups would wait forever
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes(attn_fwd_sm100)");
  if ((long long)fa.numRegs * Cfg::THREADS < 256LL * Cfg::REGS_SOFTMAX + 128LL * Cfg::REGS_OTHER)
    return fail(SA_ERR_UNSUPPORTED, "attn_fwd_sm100 launches with %d registers per thread, too few for "
                "its register split", fa.numRegs);
  kern<<<grid, Cfg::THREADS, smem, st>>>(mq, mk, mv, p);
  e = cudaGetLastError();
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "attn_fwd_sm100 launch");
}

// Backward: prep (Delta, lse2), then the dK/dV and dQ kernels, all on `st`.
template <int D, bool BF16>
int launch_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
               void* dq, void* dk, void* dv, int B, int Sq, int Sk, int Hq, int Hkv, int causal, float scale,
               float* ws, cudaStream_t st) {
  using Cfg = sa::BwdCfg<D>;
  CUtensorMap mq, mdo, mk, mv;
  int rc;
  if ((rc = make_map(&mq, q, BF16, D, Hq, Sq, B, 128)) != SA_OK) return rc;
  if ((rc = make_map(&mdo, dout, BF16, D, Hq, Sq, B, 128)) != SA_OK) return rc;
  if ((rc = make_map(&mk, k, BF16, D, Hkv, Sk, B, 128)) != SA_OK) return rc;
  if ((rc = make_map(&mv, v, BF16, D, Hkv, Sk, B, 128)) != SA_OK) return rc;
  sa::BwdParams p;
  p.o = o; p.dout = dout; p.lse = lse;
  p.sq_pad = (Sq + 127) / 128 * 128;
  p.nlse2 = ws;
  p.ndelta = ws + (size_t)B * Hq * p.sq_pad;
  p.dq = dq; p.dk = dk; p.dv = dv;
  p.B = B; p.Sq = Sq; p.Sk = Sk; p.Hq = Hq; p.Hkv = Hkv; p.G = Hq / Hkv; p.causal = causal;
  p.n_qt = p.sq_pad / 128;
  p.n_kt = (Sk + 127) / 128;
  p.c2 = scale * kLog2e;
  p.scale = scale;
  if ((long long)p.n_qt * Hq * B > 0x7fffffffLL || (long long)p.n_kt * Hkv * B > 0x7fffffffLL)
    return fail(SA_ERR_UNSUPPORTED, "backward grid too large");
  const long long prep_threads = (long long)B * p.sq_pad * Hq;
  sa::bwd_prep<D, BF16><<<(unsigned)((prep_threads + 255) / 256), 256, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "bwd_prep launch");
  // D = 64 would fit two CTAs per SM in shared memory, but each holds all 512 tensor-memory
  // columns: ask for enough shared memory to keep one
  const int smem = Cfg::SMEM_TOTAL > 120 * 1024 ? Cfg::SMEM_TOTAL : 120 * 1024;
  auto kv = sa::attn_bwd_kv<D, BF16>;
  auto kq = sa::attn_bwd_q<D, BF16>;
  if ((e = cudaFuncSetAttribute(kv, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
    return cuda_fail(e, "cudaFuncSetAttribute(attn_bwd_kv)");
  if ((e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
    return cuda_fail(e, "cudaFuncSetAttribute(attn_bwd_q)");
  kv<<<p.n_kt * Hkv * B, Cfg::THREADS, smem, st>>>(mq, mdo, mk, mv, p);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "attn_bwd_kv launch");
  kq<<<p.n_qt * Hq * B, Cfg::THREADS, smem, st>>>(mq, mdo, mk, mv, p);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "attn_bwd_q launch");
  return SA_OK;
}

template <int D, bool BF16>
int launch_simple(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Sq,
                  int Sk, int Hq, int Hkv, int causal, float scale, cudaStream_t st) {
  dim3 grid((Sq + 63) / 64, Hq, B);
  if (grid.y > 65535 || grid.z > 65535) return fail(SA_ERR_UNSUPPORTED, "Hq or B too large for the simple kernel");
  sa::attn_fwd_simple<D, BF16><<<grid, 64, 0, st>>>(q, k, v, o, lse, Sq, Sk, Hq, Hkv, causal, scale * kLog2e);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "attn_fwd_simple launch");
}

// ---------------------------------------------------------------- decode planning
size_t dec_ws_bytes(int B, int Hq, int nsplit, int D) {
  return (size_t)B * Hq * nsplit * (D + 4) * sizeof(float);
}

struct DecPlan {
  int nsplit, chunk, ngrp;
};

// max_chunk: the most tokens one split may take (paged decode: its stage table's size).
DecPlan plan_decode(int B, int Sk, int Hq, int Hkv, int D, int num_splits, int sms,
                    int max_chunk = 0x7fffffff) {
  DecPlan pl;
  const int G = Hq / Hkv;
  pl.ngrp = (G + 15) / 16;
  const long long groups = (long long)B * Hkv * pl.ngrp;
  int max_split = (Sk + 63) / 64;
  const int cap = D == 64 ? sa::DecMerge<64>::MAX_SPLITS : sa::DecMerge<128>::MAX_SPLITS;
  if (max_split > cap) max_split = cap;
  long long want = num_splits > 0 ? num_splits : (3LL * sms + groups - 1) / groups;
  if (want < 1) want = 1;
  if (want > max_split) want = max_split;
  int chunk = (int)((Sk + want - 1) / want);
  chunk = (chunk + 63) / 64 * 64;
  if (chunk > max_chunk) chunk = max_chunk;     // more splits than the cap above: caller checks
  pl.chunk = chunk;
  pl.nsplit = (Sk + chunk - 1) / chunk;
  return pl;
}

// Paged K/V caches for launch_decode: [num_pages, page_size, Hkv, D], block table
// [B, max_blocks], sequence lengths [B] (all device memory).
struct DecPaged {
  const int* block_table = nullptr;
  const int* seqlens = nullptr;
  int max_blocks = 0, page_size = 0, num_pages = 0;
};

// Arrival counters of the single-kernel decode: kDecSemSlots sets of kDecSemTiles, zero with
// the module; launches take sets in turn and every tile's last split zeroes its counter, so
// up to kDecSemSlots single-kernel decodes may be in flight at once (on any streams).
constexpr int kDecSemSlots = 16, kDecSemTiles = 4096;
static __device__ unsigned int g_dec_sem[kDecSemSlots * kDecSemTiles];

int dec_sem_slot(unsigned int** out) {
  static std::atomic<unsigned int> next{0};
  void* base = nullptr;
  int rc = device_symbol((const void*)&g_dec_sem, "decode arrival counters", &base);
  if (rc != SA_OK) return rc;
  *out = static_cast<unsigned int*>(base) + (size_t)kDecSemTiles * (next++ % kDecSemSlots);
  return SA_OK;
}

// FUSED: the single-kernel instance (the tile's last split merges; no combine launch).
template <int D, bool BF16, bool PAGED, bool FUSED = false>
int launch_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Sk,
                  int Hq, int Hkv, float scale, const DecPlan& pl, void* ws, cudaStream_t st,
                  const DecPaged& pg = DecPaged()) {
  using Cfg = sa::DecCfg<D>;
  CUtensorMap mk, mv;
  int rc;
  // TMA views: (D, Hkv, token, batch), or for a paged cache (D, Hkv, row in page, page)
  const int rows = PAGED ? pg.page_size : Sk, outer = PAGED ? pg.num_pages : B;
  if ((rc = make_map(&mk, k, BF16, D, Hkv, rows, outer, 64)) != SA_OK) return rc;
  if ((rc = make_map(&mv, v, BF16, D, Hkv, rows, outer, 64)) != SA_OK) return rc;
  sa::DecParams p;
  p.block_table = pg.block_table; p.seqlens = pg.seqlens;
  p.max_blocks = pg.max_blocks; p.page_size = pg.page_size;
  p.q = q;
  p.ws_ml = reinterpret_cast<float*>(ws);
  p.ws_o = p.ws_ml + (size_t)B * Hq * pl.nsplit * 4;
  p.o = o; p.lse = lse;
  p.B = B; p.Sk = Sk; p.Hq = Hq; p.Hkv = Hkv; p.G = Hq / Hkv; p.ngrp = pl.ngrp;
  p.nsplit = pl.nsplit; p.chunk = pl.chunk;
  p.c2 = scale * kLog2e;
  p.sem = nullptr;
  dim3 grid(pl.nsplit, Hkv * pl.ngrp, B);
  if ((long long)B * Hq > 0x7fffffffLL || grid.y > 65535 || grid.z > 65535)
    return fail(SA_ERR_UNSUPPORTED, "decode grid too large");
  if (FUSED) {
    if ((long long)B * Hkv * pl.ngrp > kDecSemTiles)
      return fail(SA_ERR_UNSUPPORTED, "single-kernel decode supports at most %d (batch, KV head, head group) "
                  "tiles (got %lld)", kDecSemTiles, (long long)B * Hkv * pl.ngrp);
    if ((rc = dec_sem_slot(&p.sem)) != SA_OK) return rc;
  }
  auto ks = sa::attn_decode_split<D, BF16, PAGED, FUSED>;
  cudaError_t e = cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_TOTAL);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attn_decode_split)");
  ks<<<grid, 128, Cfg::SMEM_TOTAL, st>>>(mk, mv, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attn_decode_split launch");
  if (FUSED) return SA_OK;
  // combine: programmatic dependent launch, resident and waiting when the split grid ends
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(B * Hq));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, sa::attn_decode_combine<D, BF16>, p);
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "attn_decode_combine launch");
}

// ---------------------------------------------------------------- built-in decode scratch
// Scratch for sa_attn_decode_noalloc: a fixed area in the library's own device image, so
// that entry point needs no memory from the caller and allocates none.  Every GPU that
// loads the library holds it until the process exits.  Host code must not use the
// symbol's name as an address: the device address is looked up once per device.
constexpr size_t kNoAllocScratchBytes = 8u << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device.  Returns SA_OK or SA_ERR_CUDA.
int noalloc_scratch(void** out) {
  return device_symbol((const void*)g_noalloc_scratch, "built-in decode scratch", out);
}

// Shared by the 16-bit and the FP8 block-sparse entry points (fp8: q, k, v e4m3, o bf16,
// scale with the Q and K descales folded in, o_mul the V descale).
int block_sparse_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                     const unsigned char* block_mask, int B, int Sq, int Sk, int Hq, int Hkv, int D, int causal,
                     float scale, int dtype, bool fp8, float o_mul, void* workspace, size_t workspace_bytes,
                     cudaStream_t st);

}  // namespace

extern "C" {

int sa_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Sq,
                int Sk, int Hq, int Hkv, int D, int causal, float scale, int dtype, sa_stream_t stream) {
  int rc = check_dims(B, Sq, Sk, Hq, Hkv, D, dtype, scale);
  if (rc != SA_OK) return rc;
  if (causal != 0 && causal != 1) return fail(SA_ERR_INVALID, "causal must be 0 or 1");
  if (B == 0 || Sq == 0 || Hq == 0) return SA_OK;
  if ((rc = check_ptrs(q, Sk ? k : q, Sk ? v : q, o, lse)) != SA_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (Sk == 0) return launch_fill(o, (size_t)B * Sq * Hq * D, lse, (size_t)B * Hq * Sq, st);
  const bool bf = dtype == SA_BF16;
  if (D == 64) return bf ? launch_fwd<64, true>(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, causal, scale, st)
                         : launch_fwd<64, false>(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, causal, scale, st);
  return bf ? launch_fwd<128, true>(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, causal, scale, st)
            : launch_fwd<128, false>(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, causal, scale, st);
}

int sa_attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                       const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int max_seqlen_q,
                       int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, int D, int causal,
                       float scale, int dtype, sa_stream_t stream) {
  int rc = check_dims(B, total_q, total_k, Hq, Hkv, D, dtype, scale);
  if (rc != SA_OK) return rc;
  if (max_seqlen_q < 0 || max_seqlen_k < 0)
    return fail(SA_ERR_INVALID, "negative max_seqlen (q %d, k %d)", max_seqlen_q, max_seqlen_k);
  if (causal != 0 && causal != 1) return fail(SA_ERR_INVALID, "causal must be 0 or 1");
  if (B == 0 || total_q == 0 || Hq == 0 || max_seqlen_q == 0) return SA_OK;
  if (!cu_seqlens_q || !cu_seqlens_k) return fail(SA_ERR_INVALID, "cu_seqlens_q and cu_seqlens_k must be non-null");
  if (((uintptr_t)cu_seqlens_q & 3u) || ((uintptr_t)cu_seqlens_k & 3u))
    return fail(SA_ERR_INVALID, "cu_seqlens pointers must be 4-byte aligned");
  if ((rc = check_ptrs(q, total_k ? k : q, total_k ? v : q, o, lse)) != SA_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (total_k == 0) return launch_fill(o, (size_t)total_q * Hq * D, lse, (size_t)Hq * total_q, st);
  FwdVarlen vl;
  vl.cu_q = cu_seqlens_q; vl.cu_k = cu_seqlens_k;
  vl.max_sq = max_seqlen_q; vl.max_sk = max_seqlen_k;
  const bool bf = dtype == SA_BF16;
  if (D == 64)
    return bf ? launch_fwd<64, true>(q, k, v, o, lse, B, total_q, total_k, Hq, Hkv, causal, scale, st, vl)
              : launch_fwd<64, false>(q, k, v, o, lse, B, total_q, total_k, Hq, Hkv, causal, scale, st, vl);
  return bf ? launch_fwd<128, true>(q, k, v, o, lse, B, total_q, total_k, Hq, Hkv, causal, scale, st, vl)
            : launch_fwd<128, false>(q, k, v, o, lse, B, total_q, total_k, Hq, Hkv, causal, scale, st, vl);
}

int sa_attn_fwd_paged(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                      const int* cu_seqlens_q, const int* block_table, const int* seqlens_k, int B,
                      int max_seqlen_q, int total_q, int Hq, int Hkv, int D, int page_size, int max_blocks,
                      int num_pages, int causal, float scale, int dtype, sa_stream_t stream) {
  int rc = check_dims(B, total_q, 1, Hq, Hkv, D, dtype, scale);
  if (rc != SA_OK) return rc;
  if (max_seqlen_q < 0) return fail(SA_ERR_INVALID, "negative max_seqlen_q");
  if (causal != 0 && causal != 1) return fail(SA_ERR_INVALID, "causal must be 0 or 1");
  if (page_size <= 0 || page_size % 128 != 0)
    return fail(SA_ERR_UNSUPPORTED, "page_size must be a positive multiple of 128 (got %d)", page_size);
  if (max_blocks <= 0 || num_pages <= 0) return fail(SA_ERR_INVALID, "max_blocks and num_pages must be positive");
  if ((long long)max_blocks * page_size > 0x7fffffffLL) return fail(SA_ERR_UNSUPPORTED, "block table too long");
  if (B == 0 || total_q == 0 || Hq == 0 || max_seqlen_q == 0) return SA_OK;
  if (!cu_seqlens_q || !block_table || !seqlens_k)
    return fail(SA_ERR_INVALID, "cu_seqlens_q, block_table and seqlens_k must be non-null");
  if (((uintptr_t)cu_seqlens_q & 3u) || ((uintptr_t)block_table & 3u) || ((uintptr_t)seqlens_k & 3u))
    return fail(SA_ERR_INVALID, "cu_seqlens_q, block_table and seqlens_k must be 4-byte aligned");
  if ((rc = check_ptrs(q, k_cache, v_cache, o, lse)) != SA_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  FwdVarlen vl;
  vl.cu_q = cu_seqlens_q;
  vl.max_sq = max_seqlen_q;
  vl.max_sk = max_blocks * page_size;
  vl.block_table = block_table; vl.seqlens_k = seqlens_k;
  vl.max_blocks = max_blocks; vl.page_size = page_size; vl.num_pages = num_pages;
  const int cap = max_blocks * page_size;
  const bool bf = dtype == SA_BF16;
  if (D == 64)
    return bf ? launch_fwd<64, true>(q, k_cache, v_cache, o, lse, B, total_q, cap, Hq, Hkv, causal, scale, st, vl)
              : launch_fwd<64, false>(q, k_cache, v_cache, o, lse, B, total_q, cap, Hq, Hkv, causal, scale, st, vl);
  return bf ? launch_fwd<128, true>(q, k_cache, v_cache, o, lse, B, total_q, cap, Hq, Hkv, causal, scale, st, vl)
            : launch_fwd<128, false>(q, k_cache, v_cache, o, lse, B, total_q, cap, Hq, Hkv, causal, scale, st, vl);
}

size_t sa_attn_fwd_block_sparse_workspace_size(int B, int Sq, int Sk, int Hq) {
  if (B <= 0 || Sq <= 0 || Sk <= 0 || Hq <= 0) return 0;
  if ((Sk + 127) / 128 > sa::kSparseMaxKTiles) return 0;
  return (size_t)B * Hq * ((Sq + 255) / 256) * sparse_stride(Sk) * sizeof(uint16_t);
}

int sa_attn_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse,
                             const unsigned char* block_mask, int B, int Sq, int Sk, int Hq, int Hkv,
                             int D, int causal, float scale, int dtype, void* workspace,
                             size_t workspace_bytes, sa_stream_t stream) {
  int rc = check_dims(B, Sq, Sk, Hq, Hkv, D, dtype, scale);
  if (rc != SA_OK) return rc;
  return block_sparse_fwd(q, k, v, o, lse, block_mask, B, Sq, Sk, Hq, Hkv, D, causal, scale, dtype, false, 1.f,
                          workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

int sa_attn_fwd_block_sparse_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                                 const unsigned char* block_mask, int B, int Sq, int Sk, int Hq, int Hkv,
                                 int D, int causal, float scale, float q_descale, float k_descale,
                                 float v_descale, void* workspace, size_t workspace_bytes, sa_stream_t stream) {
  int rc = check_dims(B, Sq, Sk, Hq, Hkv, D, SA_BF16, scale);
  if (rc != SA_OK) return rc;
  if (D != 128) return fail(SA_ERR_UNSUPPORTED, "the FP8 forward supports D = 128 (got %d)", D);
  if (!(std::isfinite(q_descale) && q_descale > 0.f && std::isfinite(k_descale) && k_descale > 0.f &&
        std::isfinite(v_descale) && v_descale > 0.f))
    return fail(SA_ERR_INVALID, "descale factors must be finite and positive");
  return block_sparse_fwd(q, k, v, o, lse, block_mask, B, Sq, Sk, Hq, Hkv, D, causal,
                          scale * q_descale * k_descale, SA_BF16, true, v_descale, workspace, workspace_bytes,
                          reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {
int block_sparse_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                     const unsigned char* block_mask, int B, int Sq, int Sk, int Hq, int Hkv, int D, int causal,
                     float scale, int dtype, bool fp8, float o_mul, void* workspace, size_t workspace_bytes,
                     cudaStream_t st) {
  int rc = SA_OK;
  if (causal != 0 && causal != 1) return fail(SA_ERR_INVALID, "causal must be 0 or 1");
  if (B == 0 || Sq == 0 || Hq == 0) return SA_OK;
  if ((rc = check_ptrs(q, Sk ? k : q, Sk ? v : q, o, lse)) != SA_OK) return rc;
  if (Sk == 0) return launch_fill(o, (size_t)B * Sq * Hq * D, lse, (size_t)B * Hq * Sq, st);
  if (!block_mask) return fail(SA_ERR_INVALID, "block_mask must be non-null");
  if ((Sk + 127) / 128 > sa::kSparseMaxKTiles)
    return fail(SA_ERR_UNSUPPORTED, "block-sparse forward supports at most %d keys (Sk=%d)",
                sa::kSparseMaxKTiles * 128, Sk);
  const size_t need = sa_attn_fwd_block_sparse_workspace_size(B, Sq, Sk, Hq);
  if (!workspace || workspace_bytes < need)
    return fail(SA_ERR_WORKSPACE, "block-sparse workspace of %zu bytes needed, %zu given", need,
                workspace ? workspace_bytes : (size_t)0);
  if (!aligned16(workspace)) return fail(SA_ERR_INVALID, "workspace must be 16-byte aligned");
  const int n_qblk = (Sq + 255) / 256;
  const long long n_rec = (long long)B * Hq * n_qblk;
  if (n_rec > 0x7fffffffLL) return fail(SA_ERR_UNSUPPORTED, "too many work units (%lld)", n_rec);
  FwdSparse sp;
  sp.sp = static_cast<const uint16_t*>(workspace);
  sp.stride = sparse_stride(Sk);
  sa::sparse_unit_lists<<<(unsigned)((n_rec + 7) / 8), 256, 0, st>>>(
      block_mask, static_cast<uint16_t*>(workspace), B, Hq, Sq, Sk, causal, n_qblk, sp.stride);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "sparse_unit_lists launch");
  const bool bf = dtype == SA_BF16;
  const FwdVarlen none;
  if (fp8) return launch_fwd<128, true, true>(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, causal, scale, st, none, sp, o_mul);
  if (D == 64)
    return bf ? launch_fwd<64, true>(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, causal, scale, st, none, sp)
              : launch_fwd<64, false>(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, causal, scale, st, none, sp);
  return bf ? launch_fwd<128, true>(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, causal, scale, st, none, sp)
            : launch_fwd<128, false>(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, causal, scale, st, none, sp);
}
}  // namespace

extern "C" {

int sa_attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Sq, int Sk,
                    int Hq, int Hkv, int D, int causal, float scale, float q_descale, float k_descale,
                    float v_descale, sa_stream_t stream) {
  int rc = check_dims(B, Sq, Sk, Hq, Hkv, D, SA_BF16, scale);
  if (rc != SA_OK) return rc;
  if (D != 128) return fail(SA_ERR_UNSUPPORTED, "the FP8 forward supports D = 128 (got %d)", D);
  if (!(std::isfinite(q_descale) && q_descale > 0.f && std::isfinite(k_descale) && k_descale > 0.f &&
        std::isfinite(v_descale) && v_descale > 0.f))
    return fail(SA_ERR_INVALID, "descale factors must be finite and positive");
  if (causal != 0 && causal != 1) return fail(SA_ERR_INVALID, "causal must be 0 or 1");
  if (B == 0 || Sq == 0 || Hq == 0) return SA_OK;
  if ((rc = check_ptrs(q, Sk ? k : q, Sk ? v : q, o, lse)) != SA_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (Sk == 0) return launch_fill(o, (size_t)B * Sq * Hq * D, lse, (size_t)B * Hq * Sq, st);
  return launch_fwd<128, true, true>(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, causal, scale * q_descale * k_descale,
                                     st, FwdVarlen(), FwdSparse(), v_descale);
}

size_t sa_attn_bwd_workspace_size(int B, int Sq, int Hq) {
  if (B <= 0 || Sq <= 0 || Hq <= 0) return 0;
  return 2 * (size_t)B * Hq * (((size_t)Sq + 127) / 128 * 128) * sizeof(float);
}

int sa_attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                void* dq, void* dk, void* dv, int B, int Sq, int Sk, int Hq, int Hkv, int D, int causal,
                float scale, int dtype, void* workspace, size_t workspace_bytes, sa_stream_t stream) {
  int rc = check_dims(B, Sq, Sk, Hq, Hkv, D, dtype, scale);
  if (rc != SA_OK) return rc;
  if (causal != 0 && causal != 1) return fail(SA_ERR_INVALID, "causal must be 0 or 1");
  if (B == 0 || Hq == 0) return SA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t kv_bytes = (size_t)B * Sk * Hkv * D * 2;
  if (Sq == 0 || Sk == 0) {
    // no (query, key) pair: every gradient is zero
    if (Sk > 0 && (!dk || !dv)) return fail(SA_ERR_INVALID, "dk and dv must be non-null");
    if (Sq > 0 && !dq) return fail(SA_ERR_INVALID, "dq must be non-null");
    cudaError_t e = cudaSuccess;
    if (Sk > 0 && e == cudaSuccess) e = cudaMemsetAsync(dk, 0, kv_bytes, st);
    if (Sk > 0 && e == cudaSuccess) e = cudaMemsetAsync(dv, 0, kv_bytes, st);
    if (Sq > 0 && e == cudaSuccess) e = cudaMemsetAsync(dq, 0, (size_t)B * Sq * Hq * D * 2, st);
    return e == cudaSuccess ? SA_OK : cuda_fail(e, "zero fill of the gradients");
  }
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv)
    return fail(SA_ERR_INVALID, "q, k, v, o, lse, dout, dq, dk and dv must be non-null");
  const void* ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return fail(SA_ERR_INVALID, "tensor pointers must be 16-byte aligned");
  const size_t need = sa_attn_bwd_workspace_size(B, Sq, Hq);
  if (!workspace || workspace_bytes < need)
    return fail(SA_ERR_WORKSPACE, "backward workspace of %zu bytes needed, %zu given", need,
                workspace ? workspace_bytes : (size_t)0);
  if (!aligned16(workspace)) return fail(SA_ERR_INVALID, "workspace must be 16-byte aligned");
  float* ws = static_cast<float*>(workspace);
  const bool bf = dtype == SA_BF16;
  if (D == 64)
    return bf ? launch_bwd<64, true>(q, k, v, o, lse, dout, dq, dk, dv, B, Sq, Sk, Hq, Hkv, causal, scale, ws, st)
              : launch_bwd<64, false>(q, k, v, o, lse, dout, dq, dk, dv, B, Sq, Sk, Hq, Hkv, causal, scale, ws, st);
  return bf ? launch_bwd<128, true>(q, k, v, o, lse, dout, dq, dk, dv, B, Sq, Sk, Hq, Hkv, causal, scale, ws, st)
            : launch_bwd<128, false>(q, k, v, o, lse, dout, dq, dk, dv, B, Sq, Sk, Hq, Hkv, causal, scale, ws, st);
}

int sa_attn_fwd_simple(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int Sq, int Sk, int Hq, int Hkv, int D, int causal, float scale, int dtype,
                       sa_stream_t stream) {
  int rc = check_dims(B, Sq, Sk, Hq, Hkv, D, dtype, scale);
  if (rc != SA_OK) return rc;
  if (causal != 0 && causal != 1) return fail(SA_ERR_INVALID, "causal must be 0 or 1");
  if (B == 0 || Sq == 0 || Hq == 0) return SA_OK;
  if ((rc = check_ptrs(q, Sk ? k : q, Sk ? v : q, o, lse)) != SA_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf = dtype == SA_BF16;
  if (D == 64) return bf ? launch_simple<64, true>(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, causal, scale, st)
                         : launch_simple<64, false>(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, causal, scale, st);
  return bf ? launch_simple<128, true>(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, causal, scale, st)
            : launch_simple<128, false>(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, causal, scale, st);
}

int sa_attn_fwd_pair(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Sq,
                     int Sk, int Hq, int Hkv, int D, int causal, float scale, int dtype, sa_stream_t stream) {
  int rc = check_dims(B, Sq, Sk, Hq, Hkv, D, dtype, scale);
  if (rc != SA_OK) return rc;
  if (D != 128) return fail(SA_ERR_UNSUPPORTED, "the CTA-pair forward supports D = 128 (got %d)", D);
  if (causal != 0 && causal != 1) return fail(SA_ERR_INVALID, "causal must be 0 or 1");
  if (B == 0 || Sq == 0 || Hq == 0) return SA_OK;
  if ((rc = check_ptrs(q, Sk ? k : q, Sk ? v : q, o, lse)) != SA_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (Sk == 0) return launch_fill(o, (size_t)B * Sq * Hq * D, lse, (size_t)B * Hq * Sq, st);
  return dtype == SA_BF16
             ? launch_fwd<128, true>(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, causal, scale, st, FwdVarlen(),
                                     FwdSparse(), 1.f, true)
             : launch_fwd<128, false>(q, k, v, o, lse, B, Sq, Sk, Hq, Hkv, causal, scale, st, FwdVarlen(),
                                      FwdSparse(), 1.f, true);
}

int sa_attn_decode_num_splits(int B, int Sk, int Hq, int Hkv, int D) {
  if (check_dims(B, 1, Sk, Hq, Hkv, D, SA_FP16, 1.f) != SA_OK) return 0;
  if (B == 0 || Hq == 0 || Sk == 0) return 1;
  return plan_decode(B, Sk, Hq, Hkv, D, 0, num_sms()).nsplit;
}

size_t sa_attn_decode_workspace_size(int B, int Sk, int Hq, int Hkv, int D, int num_splits) {
  if (num_splits < 0 || check_dims(B, 1, Sk, Hq, Hkv, D, SA_FP16, 1.f) != SA_OK) return 0;
  if (B == 0 || Hq == 0 || Sk == 0) return 0;
  DecPlan pl = plan_decode(B, Sk, Hq, Hkv, D, num_splits, num_sms());
  return dec_ws_bytes(B, Hq, pl.nsplit, D);
}

int sa_attn_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Sk,
                   int Hq, int Hkv, int D, float scale, int dtype, int num_splits, void* workspace,
                   size_t workspace_bytes, sa_stream_t stream) {
  int rc = check_dims(B, 1, Sk, Hq, Hkv, D, dtype, scale);
  if (rc != SA_OK) return rc;
  if (num_splits < 0) return fail(SA_ERR_INVALID, "num_splits must be >= 0");
  if (B == 0 || Hq == 0) return SA_OK;
  if ((rc = check_ptrs(q, Sk ? k : q, Sk ? v : q, o, lse)) != SA_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (Sk == 0) return launch_fill(o, (size_t)B * Hq * D, lse, (size_t)B * Hq, st);
  DecPlan pl = plan_decode(B, Sk, Hq, Hkv, D, num_splits, num_sms());
  const size_t need = dec_ws_bytes(B, Hq, pl.nsplit, D);
  if (!workspace || workspace_bytes < need)
    return fail(SA_ERR_WORKSPACE, "decode workspace of %zu bytes needed (got %zu)", need,
                workspace ? workspace_bytes : (size_t)0);
  if (!aligned16(workspace)) return fail(SA_ERR_INVALID, "workspace must be 16-byte aligned");
  const bool bf = dtype == SA_BF16;
  if (D == 64) return bf ? launch_decode<64, true, false>(q, k, v, o, lse, B, Sk, Hq, Hkv, scale, pl, workspace, st)
                         : launch_decode<64, false, false>(q, k, v, o, lse, B, Sk, Hq, Hkv, scale, pl, workspace, st);
  return bf ? launch_decode<128, true, false>(q, k, v, o, lse, B, Sk, Hq, Hkv, scale, pl, workspace, st)
            : launch_decode<128, false, false>(q, k, v, o, lse, B, Sk, Hq, Hkv, scale, pl, workspace, st);
}

int sa_attn_decode_single(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Sk,
                          int Hq, int Hkv, int D, float scale, int dtype, int num_splits, void* workspace,
                          size_t workspace_bytes, sa_stream_t stream) {
  int rc = check_dims(B, 1, Sk, Hq, Hkv, D, dtype, scale);
  if (rc != SA_OK) return rc;
  if (num_splits < 0) return fail(SA_ERR_INVALID, "num_splits must be >= 0");
  if (B == 0 || Hq == 0) return SA_OK;
  if ((rc = check_ptrs(q, Sk ? k : q, Sk ? v : q, o, lse)) != SA_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (Sk == 0) return launch_fill(o, (size_t)B * Hq * D, lse, (size_t)B * Hq, st);
  DecPlan pl = plan_decode(B, Sk, Hq, Hkv, D, num_splits, num_sms());
  const size_t need = dec_ws_bytes(B, Hq, pl.nsplit, D);
  if (!workspace || workspace_bytes < need)
    return fail(SA_ERR_WORKSPACE, "decode workspace of %zu bytes needed (got %zu)", need,
                workspace ? workspace_bytes : (size_t)0);
  if (!aligned16(workspace)) return fail(SA_ERR_INVALID, "workspace must be 16-byte aligned");
  const bool bf = dtype == SA_BF16;
  if (D == 64)
    return bf ? launch_decode<64, true, false, true>(q, k, v, o, lse, B, Sk, Hq, Hkv, scale, pl, workspace, st)
              : launch_decode<64, false, false, true>(q, k, v, o, lse, B, Sk, Hq, Hkv, scale, pl, workspace, st);
  return bf ? launch_decode<128, true, false, true>(q, k, v, o, lse, B, Sk, Hq, Hkv, scale, pl, workspace, st)
            : launch_decode<128, false, false, true>(q, k, v, o, lse, B, Sk, Hq, Hkv, scale, pl, workspace, st);
}

int sa_attn_decode_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                           int Sk, int Hq, int Hkv, int D, float scale, int dtype, int num_splits,
                           sa_stream_t stream) {
  int rc = check_dims(B, 1, Sk, Hq, Hkv, D, dtype, scale);
  if (rc != SA_OK) return rc;
  if (num_splits < 0) return fail(SA_ERR_INVALID, "num_splits must be >= 0");
  if (B == 0 || Hq == 0) return SA_OK;
  if ((rc = check_ptrs(q, Sk ? k : q, Sk ? v : q, o, lse)) != SA_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (Sk == 0) return launch_fill(o, (size_t)B * Hq * D, lse, (size_t)B * Hq, st);
  DecPlan pl = plan_decode(B, Sk, Hq, Hkv, D, num_splits, num_sms());
  const size_t need = dec_ws_bytes(B, Hq, pl.nsplit, D);
  if (need > kNoAllocScratchBytes)
    return fail(SA_ERR_UNSUPPORTED, "this decode needs %zu bytes of scratch; the built-in area holds %zu "
                "(use sa_attn_decode with a caller workspace, or fewer splits)", need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(&scratch)) != SA_OK) return rc;
  const bool bf = dtype == SA_BF16;
  if (D == 64) return bf ? launch_decode<64, true, false>(q, k, v, o, lse, B, Sk, Hq, Hkv, scale, pl, scratch, st)
                         : launch_decode<64, false, false>(q, k, v, o, lse, B, Sk, Hq, Hkv, scale, pl, scratch, st);
  return bf ? launch_decode<128, true, false>(q, k, v, o, lse, B, Sk, Hq, Hkv, scale, pl, scratch, st)
            : launch_decode<128, false, false>(q, k, v, o, lse, B, Sk, Hq, Hkv, scale, pl, scratch, st);
}

// Checks and plan shared by the paged-decode entry points.  Returns SA_OK and fills
// *max_seqlen and *pl, or an error code.
static int paged_plan(int B, int Hq, int Hkv, int D, int dtype, float scale, int page_size, int max_blocks,
                      int num_pages, int num_splits, int* max_seqlen, DecPlan* pl) {
  int rc = check_dims(B, 1, 0, Hq, Hkv, D, dtype, scale);
  if (rc != SA_OK) return rc;
  if (num_splits < 0) return fail(SA_ERR_INVALID, "num_splits must be >= 0");
  if (page_size <= 0 || page_size % 64 != 0)
    return fail(SA_ERR_UNSUPPORTED, "page_size must be a positive multiple of 64 (got %d)", page_size);
  if (max_blocks <= 0 || num_pages <= 0)
    return fail(SA_ERR_INVALID, "max_blocks (%d) and num_pages (%d) must be positive", max_blocks, num_pages);
  const long long msl = (long long)page_size * max_blocks;
  if (msl > 0x7fffffffLL) return fail(SA_ERR_UNSUPPORTED, "page_size * max_blocks too large");
  *max_seqlen = (int)msl;
  pl->nsplit = pl->chunk = pl->ngrp = 0;
  if (B == 0 || Hq == 0) return SA_OK;                       // nothing to plan
  // one split's stage table holds MAX_PAGED_STAGES 64-token stages
  constexpr int max_chunk = sa::DecCfg<64>::MAX_PAGED_STAGES * 64;
  *pl = plan_decode(B, *max_seqlen, Hq, Hkv, D, num_splits, num_sms(), max_chunk);
  const int cap = D == 64 ? sa::DecMerge<64>::MAX_SPLITS : sa::DecMerge<128>::MAX_SPLITS;
  if (pl->nsplit > cap)
    return fail(SA_ERR_UNSUPPORTED, "paged decode of up to %d tokens needs %d splits (at most %d)", *max_seqlen,
                pl->nsplit, cap);
  return SA_OK;
}

size_t sa_attn_decode_paged_workspace_size(int B, int Hq, int Hkv, int D, int page_size, int max_blocks,
                                           int num_splits) {
  int msl = 0;
  DecPlan pl;
  if (B <= 0 || Hq <= 0) return 0;
  if (paged_plan(B, Hq, Hkv, D, SA_FP16, 1.f, page_size, max_blocks, 1, num_splits, &msl, &pl) != SA_OK) return 0;
  return dec_ws_bytes(B, Hq, pl.nsplit, D);
}

int sa_attn_decode_paged(const void* q, const void* k_cache, const void* v_cache, const int* block_table,
                         const int* seqlens, void* o, float* lse, int B, int Hq, int Hkv, int D, int page_size,
                         int max_blocks, int num_pages, float scale, int dtype, int num_splits, void* workspace,
                         size_t workspace_bytes, sa_stream_t stream) {
  int msl = 0;
  DecPlan pl;
  int rc = paged_plan(B, Hq, Hkv, D, dtype, scale, page_size, max_blocks, num_pages, num_splits, &msl, &pl);
  if (rc != SA_OK) return rc;
  if (B == 0 || Hq == 0) return SA_OK;                       // (after the argument checks)
  if ((rc = check_ptrs(q, k_cache, v_cache, o, lse)) != SA_OK) return rc;
  if (!block_table || !seqlens) return fail(SA_ERR_INVALID, "block_table and seqlens must be non-null");
  if ((long long)num_pages * page_size * Hkv * D > (1LL << 40))
    return fail(SA_ERR_UNSUPPORTED, "K/V cache too large");
  const size_t need = dec_ws_bytes(B, Hq, pl.nsplit, D);
  if (!workspace || workspace_bytes < need)
    return fail(SA_ERR_WORKSPACE, "decode workspace of %zu bytes needed (got %zu)", need,
                workspace ? workspace_bytes : (size_t)0);
  if (!aligned16(workspace)) return fail(SA_ERR_INVALID, "workspace must be 16-byte aligned");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  DecPaged pg;
  pg.block_table = block_table; pg.seqlens = seqlens;
  pg.max_blocks = max_blocks; pg.page_size = page_size; pg.num_pages = num_pages;
  const bool bf = dtype == SA_BF16;
  if (D == 64)
    return bf ? launch_decode<64, true, true>(q, k_cache, v_cache, o, lse, B, msl, Hq, Hkv, scale, pl, workspace, st, pg)
              : launch_decode<64, false, true>(q, k_cache, v_cache, o, lse, B, msl, Hq, Hkv, scale, pl, workspace, st, pg);
  return bf ? launch_decode<128, true, true>(q, k_cache, v_cache, o, lse, B, msl, Hq, Hkv, scale, pl, workspace, st, pg)
            : launch_decode<128, false, true>(q, k_cache, v_cache, o, lse, B, msl, Hq, Hkv, scale, pl, workspace, st, pg);
}

int sa_diag_read_floor(const void* src, size_t bytes, unsigned int* sink, int mode, sa_stream_t stream) {
  if (!src || !sink) return fail(SA_ERR_INVALID, "src and sink must be non-null");
  if (!aligned16(src) || (bytes & 15u)) return fail(SA_ERR_INVALID, "src must be 16-byte aligned, bytes a multiple of 16");
  if ((uintptr_t)sink & 3u) return fail(SA_ERR_INVALID, "sink must be 4-byte aligned");
  if (mode != 0 && mode != 1) return fail(SA_ERR_UNSUPPORTED, "mode must be 0 or 1 (got %d)", mode);
  if (bytes == 0) return SA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (mode == 0) {
    sa::read_floor_ld<<<4 * num_sms(), sa::kFloorThreads, 0, st>>>(static_cast<const uint4*>(src), bytes / 16, sink);
  } else {
    const int smem = 1024 + sa::kBulkStages * sa::kBulkBytes + 64;
    e = cudaFuncSetAttribute(sa::read_floor_bulk, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(read_floor_bulk)");
    sa::read_floor_bulk<<<3 * num_sms(), 128, smem, st>>>(static_cast<const uint8_t*>(src), bytes / 16, sink);
  }
  e = cudaGetLastError();
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "read_floor launch");
}

int sa_diag_exp2_poly(const float* x, float* y, int n, sa_stream_t stream) {
  if (n < 0) return fail(SA_ERR_INVALID, "negative n");
  if (n == 0) return SA_OK;
  if (!x || !y || ((uintptr_t)x & 3u) || ((uintptr_t)y & 3u))
    return fail(SA_ERR_INVALID, "x and y must be non-null, 4-byte aligned device arrays");
  const int pairs = (n + 1) / 2;
  sa::diag_exp2_poly<<<(pairs + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "diag_exp2_poly launch");
}

const char* sa_last_error(void) { return g_err.c_str(); }

int sa_check_status(sa_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int status = 0;
  e = cudaMemcpyFromSymbol(&status, sa::g_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
  if (status != 0) {
    const int zero = 0;
    cudaMemcpyToSymbol(sa::g_status, &zero, sizeof(int));
    if ((status >> 16) == sa::kStatusBadLengths)
      return fail(SA_ERR_INVALID, "packed sequence %d (mod 65536): offsets must run forward inside the "
                  "buffers and no query length may exceed max_seqlen_q", status & 0xffff);
    return fail(SA_ERR_TIMEOUT, "a device wait expired (code %d, site %d)", status >> 16, status & 0xffff);
  }
  g_err.clear();
  return SA_OK;
}

int sa_selftest_bounded_wait(sa_stream_t stream) {
  sa::selftest_bounded_wait<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>();
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SA_OK : cuda_fail(e, "selftest_bounded_wait launch");
}

const char* sa_version(void) { return "0.1.0"; }

}  // extern "C"
