/*
 * sa_attn.h -- C ABI of the B200 (sm_100a) fused online-softmax attention library.
 *
 * What is computed (for batch b, query head h, query row i; G = Hq / Hkv):
 *   kvh = h / G                                   GQA: consecutive query heads share a
 *                                                 KV head (TurboQuant "Attention API" page,
 *                                                 compute_hybrid_attention_store, the
 *                                                 (T, H_kv, G, D) query view)
 *   visible keys j: j < Sk, and j <= i + Sk - Sq when causal (bottom-right alignment;
 *                                                 the pages use Sq == Sk only)
 *   s_j = scale * <q[b,i,h,:], k[b,j,kvh,:]>
 *   O   = sum_j softmax(s)_j * v[b,j,kvh,:]       StreamAttention page, "Kernel Design
 *   LSE = log sum_j exp(s_j)  (natural log)       (Fused Online Softmax)": one streaming
 *                                                 pass with running max, running sum and a
 *                                                 rescaled accumulator; lse = running max
 *                                                 + log(denominator)
 *   no visible key -> O = 0 and LSE = -inf        (TurboQuant page: empty KV gives zeros)
 *
 * Layouts (all contiguous, row-major, elements of `dtype` unless stated):
 *   prefill  q [B, Sq, Hq, D]   k, v [B, Sk, Hkv, D]   o [B, Sq, Hq, D]   lse [B, Hq, Sq] fp32
 *   decode   q [B, Hq, D]       k, v [B, Sk, Hkv, D]   o [B, Hq, D]       lse [B, Hq]     fp32
 *   packed   q [total_q, Hq, D] k, v [total_k, Hkv, D] o [total_q, Hq, D] lse [Hq, total_q]
 *   paged    k, v caches [num_pages, page_size, Hkv, D] with a block table per sequence
 *   FP8      q, k, v e4m3 codes (1 byte), o bf16
 *
 * Entry points: sa_attn_fwd (prefill), sa_attn_fwd_varlen (packed sequences),
 * sa_attn_fwd_paged (packed queries over a paged cache), sa_attn_fwd_block_sparse (a
 * block mask), sa_attn_fwd_fp8 and sa_attn_fwd_block_sparse_fp8 (e4m3 inputs), sa_attn_bwd
 * (dQ, dK, dV), sa_attn_decode / sa_attn_decode_single / sa_attn_decode_noalloc /
 * sa_attn_decode_paged (single-token decode), plus workspace-size queries and status.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library keeps no
 *     reference after the call returns and allocates no device memory on these paths.
 *   - Work is enqueued asynchronously on `stream` (NULL = legacy default stream); nothing
 *     synchronises.  A return of SA_OK means "validated and launched".
 *   - Pointers must be 16-byte aligned (tensor-memory-access copies need it).
 *   - Arguments are checked on the host before anything is launched; the first failing
 *     check is returned and sa_last_error() describes it.  Nothing is written then.
 *   - Every device-side wait is bounded; if one expires the kernel records it in a device
 *     status word and returns early (outputs are then undefined).  sa_check_status()
 *     reports and clears that word.
 *   - In-flight limits: every forward entry point (sa_attn_fwd and its packed, paged,
 *     block-sparse and FP8 variants) may take its work units from counters in the
 *     library's device image: at most 1024 such launches in flight per device (see
 *     sa_attn_fwd).  sa_attn_decode_single: at most 16 calls in flight.  The other
 *     entry points keep no state between calls beyond sa_attn_decode_noalloc's area.
 *   - D must be 64 or 128; dtype SA_FP16 or SA_BF16; Hq a positive multiple of Hkv.
 *   - B == 0, Sq == 0 or Hq == 0: SA_OK, nothing launched.  Sk == 0: O = 0, LSE = -inf.
 */
#ifndef SA_ATTN_H
#define SA_ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same handle type as cudaStream_t / CUstream. */
typedef struct CUstream_st* sa_stream_t;

typedef enum { SA_FP16 = 0, SA_BF16 = 1 } sa_dtype_t;

typedef enum {
    SA_OK = 0,
    SA_ERR_INVALID = -1,      /* null pointer, negative size, Hq % Hkv, misalignment, bad scale */
    SA_ERR_UNSUPPORTED = -2,  /* D not in {64,128}, unknown dtype, size beyond a stated limit */
    SA_ERR_CUDA = -3,         /* a CUDA call failed; sa_last_error() has the CUDA message */
    SA_ERR_TIMEOUT = -4,      /* a bounded device wait expired (reported by sa_check_status) */
    SA_ERR_WORKSPACE = -5     /* decode workspace missing or smaller than required */
} sa_status_t;

/*
 * Prefill / full attention forward (StreamAttention page, "Kernel Design (Fused Online
 * Softmax)"; flash-attn-volta page, flash_attn_forward with return_softmax_lse).
 *   q, k, v, o : device tensors as laid out above.
 *   lse        : device fp32 [B, Hq, Sq], or NULL to skip it.
 *   causal     : 0 or 1 (bottom-right aligned when Sq != Sk).
 *   scale      : softmax scale, used as given (finite); callers usually pass 1/sqrt(D).
 *   dtype      : SA_FP16 or SA_BF16 for q, k, v and o.
 * Runs the persistent tcgen05 (tensor-memory) kernel.
 * Concurrency: for shapes whose fixed work order would balance badly, the kernel takes its
 * work units from a counter pair in the library's device image (1024 pairs, used in turn
 * by successive launches and zeroed by each launch's end).  The packed, paged,
 * block-sparse and FP8 forwards below always do.  At most 1024 such forward launches may
 * be in flight on a device at once (on any streams or graphs); a launch that found its
 * pair still in use by the launch 1024 before it would skip or repeat work units.  A CUDA
 * graph keeps the pair it was captured with: replays of one graph must not overlap.
 */
int sa_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                int B, int Sq, int Sk, int Hq, int Hkv, int D, int causal,
                float scale, int dtype, sa_stream_t stream);

/*
 * The same forward over B sequences of different lengths packed back to back (Stem /
 * AngelSlim page, section 2: the serving backend's "varlen" path; the flash-attn-volta
 * page lists variable-length sequences among what it lacks).
 *   q, o         : device [total_q, Hq, D]; k, v : device [total_k, Hkv, D] (dtype).
 *   lse          : device fp32 [Hq, total_q], or NULL.
 *   cu_seqlens_q : device int32 [B + 1]; sequence b owns query rows
 *                  cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1 (4-byte aligned).
 *   cu_seqlens_k : device int32 [B + 1]; its key rows likewise.
 *   max_seqlen_q : an upper bound on every cu_seqlens_q[b+1] - cu_seqlens_q[b] (sizes
 *                  the work list); max_seqlen_k likewise for keys (a scheduling hint).
 *   causal       : 0 or 1, bottom-right aligned within each sequence (a query chunk
 *                  shorter than its keys sees the whole prefix).
 * Each sequence gets exactly sa_attn_fwd of its own rows.  Rows of o/lse outside every
 * sequence are not written.  The offsets stay on the device: the kernel clamps them into
 * the buffers (never reading or writing outside q/k/v/o/lse), and if they run backwards,
 * leave the buffers or give a query length above max_seqlen_q it records that in the
 * device status word, so the next sa_check_status() returns SA_ERR_INVALID (outputs of the
 * offending sequences are then undefined).  B, total_q, Hq or max_seqlen_q == 0: SA_OK,
 * nothing launched; total_k == 0: O = 0, LSE = -inf for every row.
 */
int sa_attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                       const int* cu_seqlens_q, const int* cu_seqlens_k, int B,
                       int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                       int Hq, int Hkv, int D, int causal, float scale, int dtype,
                       sa_stream_t stream);

/*
 * Forward over a paged K/V cache with packed queries (chunked prefill against cached
 * prefixes; the Stem page's serving backend names "varlen" and "paged" paths): q, o
 * [total_q, Hq, D] and lse [Hq, total_q] as sa_attn_fwd_varlen (cu_seqlens_q, max_seqlen_q);
 * k_cache, v_cache [num_pages, page_size, Hkv, D]; sequence b's key t sits in page
 * block_table[b * max_blocks + t / page_size] (int32, device) at row t % page_size, its key
 * count seqlens_k[b] (int32, device; clamped to [0, page_size * max_blocks]).  Causal is
 * bottom-right aligned within each sequence.  page_size must be a positive multiple of
 * 128 (SA_ERR_UNSUPPORTED).  A table entry outside [0, num_pages) reads zeros.
 */
int sa_attn_fwd_paged(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                      const int* cu_seqlens_q, const int* block_table, const int* seqlens_k, int B,
                      int max_seqlen_q, int total_q, int Hq, int Hkv, int D, int page_size,
                      int max_blocks, int num_pages, int causal, float scale, int dtype,
                      sa_stream_t stream);

/*
 * Block-sparse forward (Stem / AngelSlim page, section 2.3: attention over the 128 x 128
 * blocks a top-k mask keeps, with the initial "sink" blocks and a sliding window of blocks
 * among them).  Same tensors, layouts and rules as sa_attn_fwd, plus:
 *   block_mask : device uint8 [B, Hq, ceil(Sq/128), ceil(Sk/128)], row-major; nonzero =
 *                query block i attends key block j.  Key j is visible to query row i iff
 *                sa_attn_fwd's rule allows it (causal: bottom-right) AND the mask keeps
 *                block (i / 128, j / 128).  A row with no visible key: O = 0, LSE = -inf.
 *   workspace  : device scratch of sa_attn_fwd_block_sparse_workspace_size() bytes,
 *                16-byte aligned, no initial contents; it receives each work unit's list
 *                of kept key blocks (a first kernel builds it from the mask).
 * Kept blocks wholly past the causal diagonal cost nothing.  Sk <= 131072 (else
 * SA_ERR_UNSUPPORTED); workspace missing or short: SA_ERR_WORKSPACE.
 */
size_t sa_attn_fwd_block_sparse_workspace_size(int B, int Sq, int Sk, int Hq);
int sa_attn_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse,
                             const unsigned char* block_mask, int B, int Sq, int Sk, int Hq,
                             int Hkv, int D, int causal, float scale, int dtype,
                             void* workspace, size_t workspace_bytes, sa_stream_t stream);

/*
 * FP8 block-sparse forward (the Stem page's serving backend: fp8 block-sparse prefill):
 * sa_attn_fwd_block_sparse on e4m3 inputs with per-tensor descales, bf16 output, D = 128;
 * inputs, outputs and descales as sa_attn_fwd_fp8, mask and workspace as
 * sa_attn_fwd_block_sparse.
 */
int sa_attn_fwd_block_sparse_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                                 const unsigned char* block_mask, int B, int Sq, int Sk, int Hq,
                                 int Hkv, int D, int causal, float scale, float q_descale,
                                 float k_descale, float v_descale, void* workspace,
                                 size_t workspace_bytes, sa_stream_t stream);

/*
 * Single-kernel split-KV decode (the StreamAttention page, "Engine Direction": the
 * two-kernel prototype loses to launch and merge overhead at small batch).  Same arguments,
 * workspace and result as sa_attn_decode; instead of a second (combine) launch, the last
 * split CTA of each (batch, KV head, head group) tile -- found by an arrival counter --
 * merges that tile's query heads.  At most 4096 such tiles (else SA_ERR_UNSUPPORTED).  The
 * arrival counters are 16 sets in the library's device image, used in turn by successive
 * calls and zeroed by each tile's merge: up to 16 calls may be in flight on a device at once
 * (any streams or graphs); replays of one captured graph must not overlap.
 */
int sa_attn_decode_single(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int Sk, int Hq, int Hkv, int D, float scale, int dtype,
                          int num_splits, void* workspace, size_t workspace_bytes,
                          sa_stream_t stream);

/*
 * FP8 forward (the Stem page's fp8 prefill path; the StreamAttention page's FP8 roadmap
 * item): q, k, v are e4m3 codes (one byte per element, layouts as sa_attn_fwd) with
 * per-tensor descale factors, o is bf16 [B, Sq, Hq, D], lse fp32 [B, Hq, Sq] or NULL.
 * Computes sa_attn_fwd of the dequantised tensors q*q_descale, k*k_descale, v*v_descale:
 * S on kind::f8f6f4 tensor cores (exact products, fp32 sums), P rounded to e4m3 for P V.
 * D must be 128 (else SA_ERR_UNSUPPORTED); descales finite and > 0 (else SA_ERR_INVALID).
 * Accuracy: each weight p = 2^(s - m_ref + 8) is rounded to e4m3 against its row's running
 * reference max m_ref, which moves whenever the row max passes it by 0.75 (log2 units),
 * so the largest weights sit near 2^8 (under e4m3's 448) and only weights below 2^-18 of the
 * row max round to zero.  O is normalised by the sum of the rounded weights; the LSE comes
 * from fp32 sums of the unrounded ones (the offset taken off), as in sa_attn_fwd.
 */
int sa_attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                    int B, int Sq, int Sk, int Hq, int Hkv, int D, int causal, float scale,
                    float q_descale, float k_descale, float v_descale, sa_stream_t stream);

/*
 * Attention backward: dQ, dK, dV of the forward's O for an upstream gradient dO
 * (StreamAttention page, "Backward": the QK tiles are recomputed from the saved LSE and
 * dQ/dK/dV are streamed, never the attention matrix; flash-attn-volta page, backward).
 *   q, k, v, causal, scale, dtype : as given to sa_attn_fwd;
 *   o, lse     : that forward's output [B, Sq, Hq, D] and LSE [B, Hq, Sq] (fp32, required);
 *   dout       : [B, Sq, Hq, D] upstream gradient (dtype);
 *   dq         : out [B, Sq, Hq, D]; dk, dv : out [B, Sk, Hkv, D] (dtype; dk and dv summed
 *                over the query heads that share a KV head);
 *   workspace  : device scratch of sa_attn_bwd_workspace_size() bytes, 16-byte aligned,
 *                no initial contents (per-row Delta = rowsum(dout * o) and LSE * log2 e).
 * Rows without a visible key contribute nothing.  Sq == 0 or Sk == 0: the gradients are
 * zero-filled.  Three kernels on `stream`; no atomics, deterministic.
 */
size_t sa_attn_bwd_workspace_size(int B, int Sq, int Hq);
int sa_attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                const void* dout, void* dq, void* dk, void* dv, int B, int Sq, int Sk, int Hq,
                int Hkv, int D, int causal, float scale, int dtype, void* workspace,
                size_t workspace_bytes, sa_stream_t stream);

/*
 * Bytes of decode workspace needed for `num_splits` (0 = the automatic choice):
 * B * Hq * splits * (D + 4) * 4.  It holds, per (b, h, split), the split's running max
 * and two running sums (of the 16-bit weights the MMA used, and of the fp32 weights for
 * the LSE) padded to 4 floats, then its unnormalised fp32 output row -- the partial
 * online-softmax states of the StreamAttention page, "Engine Direction".
 * Returns 0 for empty problems or invalid sizes.
 */
size_t sa_attn_decode_workspace_size(int B, int Sk, int Hq, int Hkv, int D, int num_splits);

/* The split count sa_attn_decode uses for num_splits = 0 on the current device (>= 1),
 * or 0 for invalid sizes. */
int sa_attn_decode_num_splits(int B, int Sk, int Hq, int Hkv, int D);

/*
 * Single-token split-KV decode with an LSE-weighted combine (StreamAttention page,
 * "Engine Direction" and "Distributed and Long-Context Variants": partial states merged
 * with log-sum-exp weights).
 *   q [B, Hq, D], k/v [B, Sk, Hkv, D], o [B, Hq, D]; lse [B, Hq] fp32 or NULL.
 *   num_splits : KV splits per (b, kv head); 0 = automatic; clamped to ceil(Sk / 64) and
 *                to 192 (D = 64) / 96 (D = 128).
 *   workspace  : device buffer of at least sa_attn_decode_workspace_size(...) bytes,
 *                16-byte aligned, owned by the caller; scratch (no initial contents
 *                needed, overwritten); calls that may run concurrently must not share it.
 * Launches the split kernel and, with programmatic dependent launch on the same stream,
 * the combine kernel (one CTA per (b, h)) that merges the splits with log-sum-exp weights.
 */
int sa_attn_decode(const void* q, const void* k, const void* v, void* o, float* lse,
                   int B, int Sk, int Hq, int Hkv, int D, float scale, int dtype,
                   int num_splits, void* workspace, size_t workspace_bytes,
                   sa_stream_t stream);

/*
 * The same decode as sa_attn_decode, for callers that cannot hand the library any device
 * memory for scratch: runtimes that reserve all GPU memory up front and forbid further
 * allocation, or hosts whose allocator is not reachable from the code that issues the
 * call.  (The pages have no counterpart; this is a deployment convenience.)
 *   Arguments as for sa_attn_decode, minus the workspace.  The scratch is a fixed 8 MiB
 *   area inside the library's device image, present on every GPU that loads the library
 *   until the process exits; this call allocates nothing (no cudaMalloc, cudaFree or
 *   allocating library routine).
 *   Limit: the split states must fit, B * Hq * splits * (D + 4) * 4 <= 8 MiB (splits as
 *   chosen by num_splits, see sa_attn_decode_workspace_size); larger problems return
 *   SA_ERR_UNSUPPORTED and leave the outputs untouched.
 *   The area is part of the library's device code, which the CUDA runtime loads onto a
 *   device when the library first uses it there (lazy module loading is the default):
 *   the first call into the library on a device -- this entry point or any other --
 *   takes the area's 8 MiB of device memory then.  A runtime that reserves the rest of
 *   GPU memory afterwards must make one library call on each device before reserving.
 *   The first call of this entry point on a device also looks up the area's device
 *   address (with that device current) and caches it for the device's current context;
 *   make that first call before any stream capture.
 *   Every call uses the same area: calls whose work may overlap on the GPU (other
 *   streams, other host threads) race and give undefined results.  Nothing in the area
 *   needs to start at zero; each call writes every byte it reads.
 */
int sa_attn_decode_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                           int B, int Sk, int Hq, int Hkv, int D, float scale, int dtype,
                           int num_splits, sa_stream_t stream);

/*
 * Single-token decode over a paged K/V cache, sequences of their own lengths: the paged
 * layout of the Stem (AngelSlim sparse attention) page's serving backend (section 2: its
 * prefill has "varlen" and "paged" paths) applied to the split-KV decode above; the
 * flash-attn-volta page ("What's NOT here") lists variable-length sequences as missing.
 * For sequence b the keys are tokens 0 .. seqlens[b]-1; token t lives in cache page
 * block_table[b * max_blocks + t / page_size] at row t % page_size.  The result is the
 * attention of q[b] over those keys, as sa_attn_decode computes it over a dense K/V.
 *   q [B, Hq, D], o [B, Hq, D] (dtype); lse [B, Hq] fp32 or NULL.
 *   k_cache, v_cache : [num_pages, page_size, Hkv, D] (dtype), 16-byte aligned.
 *   block_table : [B, max_blocks] int32, device memory; entries for the tokens in use must
 *                 be in [0, num_pages) (others are never read).
 *   seqlens     : [B] int32, device memory; values are clamped to [0, page_size * max_blocks].
 *                 A sequence of length 0 gives O = 0, LSE = -inf.
 *   page_size   : a positive multiple of 64 (SA_ERR_UNSUPPORTED otherwise).
 *   num_splits  : as for sa_attn_decode, planned for page_size * max_blocks tokens; a split
 *                 covers at most 16384 tokens, so the longest sequence may hold up to
 *                 192 * 16384 (D = 64) / 96 * 16384 (D = 128) tokens.
 *   workspace   : at least sa_attn_decode_paged_workspace_size(...) bytes, rules as for
 *                 sa_attn_decode.
 * Errors as for sa_attn_decode, plus SA_ERR_INVALID for a null block_table or seqlens or
 * non-positive max_blocks / num_pages.
 */
int sa_attn_decode_paged(const void* q, const void* k_cache, const void* v_cache,
                         const int* block_table, const int* seqlens, void* o, float* lse,
                         int B, int Hq, int Hkv, int D, int page_size, int max_blocks,
                         int num_pages, float scale, int dtype, int num_splits,
                         void* workspace, size_t workspace_bytes, sa_stream_t stream);

/* Bytes of workspace sa_attn_decode_paged needs for these sizes and num_splits (0 for
 * invalid sizes or B * Hq == 0). */
size_t sa_attn_decode_paged_workspace_size(int B, int Hq, int Hkv, int D, int page_size,
                                           int max_blocks, int num_splits);

/*
 * Diagnostic only: the same forward as sa_attn_fwd computed by a plain CUDA-core kernel
 * (one thread per query row, fp32 online softmax).  Slow; used to cross-check the
 * tensor-core path.  Same arguments and conventions as sa_attn_fwd.
 */
int sa_attn_fwd_simple(const void* q, const void* k, const void* v, void* o, float* lse,
                       int B, int Sq, int Sk, int Hq, int Hkv, int D, int causal,
                       float scale, int dtype, sa_stream_t stream);

/*
 * Diagnostic: reads `bytes` of device memory at `src` once, with no attention arithmetic,
 * and XORs it into *sink (device uint32, 4-byte aligned).  mode 0: 128-bit loads from four
 * 256-thread blocks per SM, eight loads in flight per thread; mode 1: bulk asynchronous
 * copies of 16 KB into a four-stage shared-memory ring, three blocks per SM -- the way the
 * decode's split kernel streams K/V.  Gives the time one cold read of a buffer takes on
 * this GPU, the floor of a kernel bound by reading those bytes (the decode's K/V).
 * src 16-byte aligned and bytes a multiple of 16, sink non-null (else SA_ERR_INVALID);
 * mode 0 or 1 (else SA_ERR_UNSUPPORTED).  bytes == 0: SA_OK, nothing launched.
 */
int sa_diag_read_floor(const void* src, size_t bytes, unsigned int* sink, int mode,
                       sa_stream_t stream);

/*
 * Diagnostic: y[i] = 2^x[i] for i < n, computed by the FMA-pipe exponential the forward
 * kernel uses for one exponential pair in four (range reduction to x = n + f, |f| <= 1/2,
 * and a fitted cubic for 2^f; arguments below -126 are clamped there).  x, y: device
 * float arrays of n elements (4-byte aligned).  For testing that exponential on its own.
 */
int sa_diag_exp2_poly(const float* x, float* y, int n, sa_stream_t stream);

/*
 * The same forward as sa_attn_fwd on a second kernel that runs each unit of 256 query rows
 * on a pair of CTAs (a two-CTA cluster): 2-SM tensor-core products (each SM loads half of
 * every K/V tile), S double-buffered in tensor memory so the softmax never waits for its
 * own tile's next S, the softmax of each row split over two threads.  D = 128 only (else
 * SA_ERR_UNSUPPORTED); dense layout; static work order.  Same arguments, conventions and
 * results as sa_attn_fwd -- the two kernels give identical bits.  sa_attn_fwd does not use
 * it: on this hardware both are bound by the softmax's exponentials per SM, and the pair's
 * cross-CTA hand-offs made it about 20 % slower on the shapes measured.
 */
int sa_attn_fwd_pair(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int Sq, int Sk, int Hq, int Hkv, int D, int causal,
                     float scale, int dtype, sa_stream_t stream);

/* Thread-local description of the last non-OK return of this thread ("" if none). */
const char* sa_last_error(void);

/* Synchronises `stream`, then reads and clears the device status word: SA_ERR_TIMEOUT if a
 * device wait expired since the last check, SA_ERR_INVALID if a kernel found invalid
 * packed sequence offsets (sa_attn_fwd_varlen), SA_ERR_CUDA on a CUDA error, else SA_OK. */
int sa_check_status(sa_stream_t stream);

/* Diagnostic: launches one kernel whose single bounded wait can never be satisfied, to
 * exercise failure detection without a GPU fault: after about 2 s the wait gives up, the
 * device status word records a timeout and the kernel returns.  The next
 * sa_check_status(stream) then returns SA_ERR_TIMEOUT (and clears the word); the context
 * stays usable.  Returns SA_OK once launched. */
int sa_selftest_bounded_wait(sa_stream_t stream);

/* Library version, "major.minor.patch". */
const char* sa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SA_ATTN_H */
