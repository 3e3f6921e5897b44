/*
 * libgqa: one grouped-query-attention (GQA) decode step on NVIDIA B200 (sm_100a).
 *
 * The operation is Algorithm 2 ("GQA 解码，第 t 步，单层") of the reading notes "GQA 阅读笔记"
 * (zhongzhuzhou.org, section "GQA 架构"), split into the two calls below:
 *
 *   gqa_kv_append  the lines that write this step's key/value vectors into the cache
 *                  (K_cache[t, g, :] = k_g_new, V_cache[t, g, :] = v_g_new, for every group g);
 *   gqa_decode     the per-head lines: head h reads the cache of its group g(h), scores
 *                  q_h . K_cache[:t+1, g]^T * scale, takes a softmax over those t+1 scores and
 *                  returns the weighted sum of V_cache[:t+1, g].
 *
 * With H_q query heads and H_kv key/value heads (H_kv = G, the number of groups), query heads
 * are grouped in contiguous blocks of r = H_q / H_kv: query head h (0-indexed) uses key/value
 * head h / r.  That is the page's 1-indexed g(h) = ceil(h / (H/G)).  H_kv = H_q is multi-head
 * attention (Algorithm 1 of the same page), H_kv = 1 is multi-query attention.  The lesson
 * "r-tf2-gqa" (ttlab.hopto.org) requires H_q to be a multiple of H_kv; other shapes are
 * rejected.
 *
 * Conventions shared by every call:
 *   - All tensors are dense, row-major, with the last dimension contiguous:
 *       q        [B][H_q][d]           k_new, v_new [B][H_kv][d]
 *       k_cache  [B][L_max][H_kv][d]   v_cache      [B][L_max][H_kv][d]
 *       out      [B][H_q][d]  float32 (always float32, whatever the input dtype)
 *       seq_lens [B]          int32
 *     Every pointer is a DEVICE pointer except where a comment says otherwise.
 *   - d is 64 or 128.  q, k_new, v_new and the caches share one element type (gqa_dtype_t).
 *   - Device pointers must be 16-byte aligned; `workspace` must be 256-byte aligned.
 *   - The caller owns and allocates every buffer, including the decode workspace.  The
 *     library calls no device allocator and keeps no per-call state; its only device memory
 *     is the fixed scratch array behind gqa_decode_noalloc.
 *   - Calls are asynchronous on `stream` (0 = the legacy default stream) and never
 *     synchronize the host.  Errors the host can see (a NULL pointer, a bad shape, a
 *     misaligned pointer, a short workspace) return a negative GQA_ERR_* code before anything
 *     is launched.  Errors only the device can see set bits in *status (GQA_STATUS_*, combined
 *     with atomicOr; `status` may be NULL) and skip the offending work; kernels never trap.
 *   - A non-zero return of GQA_ERR_CUDA means a CUDA runtime call failed; the CUDA error is
 *     left for cudaGetLastError().
 */
#ifndef GQA_H
#define GQA_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element type of q, k_new, v_new, k_cache and v_cache. */
typedef enum {
    GQA_DTYPE_F32 = 0,  /* IEEE float32; computed on CUDA cores in float32 */
    GQA_DTYPE_BF16 = 1, /* bfloat16; products on tcgen05 tensor cores, float32 accumulation */
    GQA_DTYPE_E4M3 = 2  /* FP8 cache (the *_fp8 calls only): e4m3 codes with per-head scales,
                           bfloat16 q; accepted by gqa_decode_workspace_size */
} gqa_dtype_t;

/* Return codes. */
#define GQA_OK 0
#define GQA_ERR_NULL (-1)                 /* a required pointer is NULL */
#define GQA_ERR_SHAPE (-2)                /* a size is not positive or too large */
#define GQA_ERR_HEADS_NOT_DIVISIBLE (-3)  /* H_q is not a multiple of H_kv */
#define GQA_ERR_UNSUPPORTED_DIM (-4)      /* d is not 64 or 128 */
#define GQA_ERR_UNSUPPORTED_DTYPE (-5)    /* dtype is not a gqa_dtype_t value */
#define GQA_ERR_ALIGNMENT (-6)            /* a pointer is not aligned as required */
#define GQA_ERR_WORKSPACE (-7)            /* workspace NULL or smaller than required */
#define GQA_ERR_CUDA (-8)                 /* a CUDA runtime call failed */
#define GQA_ERR_NO_DEVICE (-9)            /* no usable sm_100 device is current */
#define GQA_ERR_SCRATCH_LIMIT (-10)       /* gqa_decode_noalloc: the sizes need more scratch than
                                             GQA_NOALLOC_SCRATCH_BYTES */
#define GQA_ERR_OVERLAP (-11)             /* gqa_kv_append_decode: seq_lens and seq_lens_out
                                             overlap */

/* Device-side status bits (OR-ed into *status). */
#define GQA_STATUS_APPEND_OVERFLOW 1  /* gqa_kv_append: seq_lens[b] < 0 or >= L_max; row skipped */
#define GQA_STATUS_SEQLEN_RANGE 2     /* gqa_decode: seq_lens[b] < 0 or > L_max; out[b] = 0 */
#define GQA_STATUS_WAIT_TIMEOUT 4     /* gqa_decode: a pipeline wait ran past its time limit;
                                         the affected outputs are not valid */
#define GQA_STATUS_INTERNAL 8         /* gqa_decode: shared-memory base not 1024-byte aligned */
#define GQA_STATUS_PAGE_RANGE 16      /* paged calls: a block-table entry a row needs is outside
                                         [0, n_pages); page 0 was read instead, the affected
                                         outputs are not valid */

/*
 * gqa_kv_append: write this step's key and value vectors into the cache.
 *
 * Algorithm 2 of "GQA 阅读笔记", the lines that write the new rows (and Algorithm 1's for
 * MHA): for every sequence b and key/value head j, with t = seq_lens[b] on entry,
 *     k_cache[b][t][j][:] = k_new[b][j][:],  v_cache[b][t][j][:] = v_new[b][j][:],
 * then seq_lens[b] = t + 1.  The copy is bit-exact.  A sequence with t < 0 or t >= L_max is
 * left untouched (cache and length) and sets GQA_STATUS_APPEND_OVERFLOW.
 *
 *   k_new, v_new  [B][H_kv][d] device, read
 *   k_cache, v_cache [B][L_max][H_kv][d] device, written at row t only
 *   seq_lens      [B] int32 device, read and incremented
 *   status        int32 device or NULL
 * Returns GQA_OK or a GQA_ERR_* code.
 */
int gqa_kv_append(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                  int32_t *seq_lens, int B, int H_kv, int d, int L_max, gqa_dtype_t dtype,
                  int32_t *status, cudaStream_t stream);

/*
 * gqa_decode_workspace_size: bytes of device workspace gqa_decode needs for these sizes on
 * the CURRENT device (the count depends on its number of SMs).  Returns 0 when the sizes are
 * invalid or no device is current.
 */
size_t gqa_decode_workspace_size(int B, int H_q, int H_kv, int d, gqa_dtype_t dtype);

/*
 * gqa_decode: the attention of one decode step, for every sequence and query head.
 *
 * Algorithm 2 of "GQA 阅读笔记", the per-head lines; with n = seq_lens[b] (the number of
 * cached rows, already counting this step's appended row) and r = H_q / H_kv:
 *     out[b][h][:] = sum_{t<n} softmax_t( scale * q[b][h] . k_cache[b][t][h/r] )
 *                    * v_cache[b][t][h/r][:]
 * Cache rows at or beyond n are never read.  n = 0 gives out[b] = 0 (a softmax over no rows
 * is undefined; zero is this library's convention).  n < 0 or n > L_max gives out[b] = 0
 * and sets GQA_STATUS_SEQLEN_RANGE.  Each cached K/V row is read from memory once per group
 * and serves all r query heads of the group.
 *
 *   q          [B][H_q][d] device, read
 *   k_cache, v_cache [B][L_max][H_kv][d] device, read (rows < seq_lens[b] only)
 *   seq_lens   [B] int32 device, read
 *   scale      softmax scale, usually 1/sqrt(d)
 *   out        [B][H_q][d] float32 device, written
 *   workspace  device scratch of at least gqa_decode_workspace_size() bytes, 256-byte aligned;
 *              owned by the caller.  It must be zero-filled once before its first use
 *              (cudaMemset): it holds per-unit counters that every completed call leaves at
 *              zero again.  After a call that reported GQA_STATUS_WAIT_TIMEOUT, zero it again.
 *              Two calls that may run at the same time must not share one workspace.
 *   status     int32 device or NULL
 * Launches one kernel on `stream`: a split-KV pass whose CTAs merge the pieces of a split
 * sequence themselves (log-sum-exp combine by the CTA that finishes the last piece).
 * Returns GQA_OK or a GQA_ERR_* code.
 */
int gqa_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *seq_lens,
               int B, int H_q, int H_kv, int d, int L_max, float scale, gqa_dtype_t dtype,
               float *out, void *workspace, size_t workspace_bytes, int32_t *status,
               cudaStream_t stream);

/*
 * gqa_kv_append_decode: the whole of Algorithm 2 of "GQA 阅读笔记" (append, then attend over the
 * t + 1 rows) in ONE kernel launch: the result of gqa_kv_append followed by gqa_decode, bit for
 * bit, with the lengths kept in two arrays instead of incremented in place.  With
 * t = seq_lens[b] on entry:
 *   - 0 <= t < L_max: k_new[b] / v_new[b] are written to row t of the caches (bit-exact), the
 *     decode attends rows [0, t + 1), and seq_lens_out[b] = t + 1;
 *   - otherwise the row is not written (GQA_STATUS_APPEND_OVERFLOW) and the decode attends t
 *     rows as gqa_decode would (t = L_max: all of them; t < 0 or t > L_max: out[b] = 0 and
 *     GQA_STATUS_SEQLEN_RANGE); seq_lens_out[b] = t.
 * seq_lens is only read (every CTA of the kernel reads it, so it cannot change during the
 * call); seq_lens_out [B] int32 device is only written, and the two must not overlap
 * (GQA_ERR_OVERLAP).  A decode loop passes the two arrays alternately.  Only one CTA of the
 * kernel writes each appended row, just before that row's tile is copied for the decode, so
 * the row reaches the cache and the attention in the same pass; no other row of the cache is
 * written.  bfloat16 only (GQA_ERR_UNSUPPORTED_DTYPE otherwise); the workspace is that of
 * gqa_decode (gqa_decode_workspace_size), with the same zero-fill rule.  Other arguments, layouts
 * and errors as gqa_kv_append and gqa_decode.
 */
int gqa_kv_append_decode(const void *q, const void *k_new, const void *v_new, void *k_cache,
                         void *v_cache, const int32_t *seq_lens, int32_t *seq_lens_out, int B,
                         int H_q, int H_kv, int d, int L_max, float scale, gqa_dtype_t dtype,
                         float *out, void *workspace, size_t workspace_bytes, int32_t *status,
                         cudaStream_t stream);

/*
 * gqa_decode_window: gqa_decode with a sliding window.  Each query head of sequence b attends
 * only the last `window` cached rows, [max(0, n - window), n), n = seq_lens[b]; the rows before
 * them are not read.  "GQA 阅读笔记", section on what came after GQA (the Mistral 7B paragraph:
 * every token attends only the previous W = 4096 tokens, which bounds the cache a step reads by
 * W instead of L); "从MHA到GQA" lists sliding-window attention among the methods that combine
 * with GQA.  window must be >= 1 (GQA_ERR_SHAPE otherwise); window >= n is the full decode.
 * Every other argument, layout and error is that of gqa_decode, and it uses the same
 * workspace size.
 */
int gqa_decode_window(const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *seq_lens, int B, int H_q, int H_kv, int d, int L_max,
                      int window, float scale, gqa_dtype_t dtype, float *out, void *workspace,
                      size_t workspace_bytes, int32_t *status, cudaStream_t stream);

/*
 * Several query tokens per sequence (speculative decoding).  "GQA 阅读笔记", what came after GQA
 * and the engineering notes on speculative decoding: when the target model checks k drafted
 * tokens in one pass, the cache is read once and all k new queries attend it.  With Q tokens
 * per sequence, the Q new tokens are the last Q rows of the cache and token j (0 <= j < Q)
 * attends rows [0, n - Q + 1 + j) of its sequence, n = seq_lens[b] (causal among the drafts;
 * Q = 1 is gqa_decode).  Each cached K/V row is read once for all Q tokens and all r heads.
 *
 * gqa_kv_append_multi: append Q rows per sequence: k_new, v_new [B][Q][H_kv][d] go to rows
 *   t .. t+Q-1, t = seq_lens[b]; then seq_lens[b] = t + Q.  t + Q > L_max (or t < 0) is
 *   refused with GQA_STATUS_APPEND_OVERFLOW.
 * gqa_decode_multi: q [B][Q][H_q][d] -> out [B][Q][H_q][d] (float32); seq_lens[b] >= Q, else
 *   out[b] = 0 and GQA_STATUS_SEQLEN_RANGE.  1 <= Q <= 32.  The workspace is
 *   gqa_decode_multi_workspace_size(B, Q, ...) bytes.  Other arguments as gqa_decode.
 */
int gqa_kv_append_multi(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                        int32_t *seq_lens, int B, int Q, int H_kv, int d, int L_max,
                        gqa_dtype_t dtype, int32_t *status, cudaStream_t stream);
size_t gqa_decode_multi_workspace_size(int B, int Q, int H_q, int H_kv, int d, gqa_dtype_t dtype);
int gqa_decode_multi(const void *q, const void *k_cache, const void *v_cache,
                     const int32_t *seq_lens, int B, int Q, int H_q, int H_kv, int d, int L_max,
                     float scale, gqa_dtype_t dtype, float *out, void *workspace,
                     size_t workspace_bytes, int32_t *status, cudaStream_t stream);

/*
 * Paged KV cache.  "GQA 阅读笔记", section on what came after GQA (the vLLM PagedAttention
 * paragraph: the KV cache is managed in fixed-size blocks) and "GQA 深入理解", section 8
 * (PagedAttention organises the cache to cut fragmentation).  All sequences share one pool
 *     k_pool, v_pool  [n_pages][page_size][H_kv][d]
 * and block_table [B][max_pages] (int32, device) names, for every sequence b, the page holding
 * its rows [j*page_size, (j+1)*page_size): row t of sequence b is
 *     k_pool[block_table[b][t / page_size]][t % page_size].
 * Only the entries covering rows < seq_lens[b] (after the append: < seq_lens[b] + 1) are read.
 * page_size must be a multiple of 8 and, for bf16, divide the kernel's tile of T rows or be a
 * multiple of it (T = 256 for d = 64 with groups of up to 8 query heads, else 128).  A
 * sequence's capacity is max_pages * page_size rows (the L_max of the contiguous calls).
 *
 * gqa_kv_append_paged: the append of gqa_kv_append into the pool: row t = seq_lens[b] goes to
 * page block_table[b][t / page_size], row t % page_size; then seq_lens[b] = t + 1.  A full
 * sequence, or a page index outside [0, n_pages), is skipped with GQA_STATUS_APPEND_OVERFLOW.
 *
 * gqa_decode_paged: gqa_decode over the paged cache; same q, out, scale, workspace (the same
 * gqa_decode_workspace_size) and errors.  An out-of-range page index sets GQA_STATUS_PAGE_RANGE.
 */
int gqa_kv_append_paged(const void *k_new, const void *v_new, void *k_pool, void *v_pool,
                        const int32_t *block_table, int max_pages, int32_t *seq_lens, int B,
                        int H_kv, int d, int page_size, int n_pages, gqa_dtype_t dtype,
                        int32_t *status, cudaStream_t stream);
int gqa_decode_paged(const void *q, const void *k_pool, const void *v_pool,
                     const int32_t *block_table, int max_pages, const int32_t *seq_lens, int B,
                     int H_q, int H_kv, int d, int page_size, int n_pages, float scale,
                     gqa_dtype_t dtype, float *out, void *workspace, size_t workspace_bytes,
                     int32_t *status, cudaStream_t stream);

/*
 * FP8 (e4m3) KV cache with one scale per key/value head.  "GQA 阅读笔记", section
 * "复现性与工程实践", mixed-precision item: serving systems store the KV cache in FP8, which
 * halves the per-step KV bytes of a 16-bit cache (GQA-8 with FP8 reads 16x fewer bytes than
 * MHA with FP16); the FlashAttention-2 GQA article (intelliparadigm.com), section 4.2 item 3,
 * stores the cache in FP8 and dequantises it when read.  The pages fix neither the format nor
 * the scaling; this library reads them as:
 *   - the cache holds OCP FP8 E4M3 codes (1 sign, 4 exponent bits with bias 7, 3 mantissa
 *     bits, no infinities, 0x7F / 0xFF NaN, largest finite magnitude 448), one byte per element,
 *     in the layouts of the 16-bit calls: k_cache, v_cache [B][L_max][H_kv][d] uint8, or the
 *     paged pools [n_pages][page_size][H_kv][d] uint8;
 *   - k_scale, v_scale [H_kv] float32 (device): code c of key/value head g stands for
 *     value(c) * k_scale[g] in K and value(c) * v_scale[g] in V;
 *   - q is bfloat16 [B][H_q][d]; out is float32.
 *
 * gqa_kv_append_fp8 / gqa_kv_append_paged_fp8: the append of gqa_kv_append / gqa_kv_append_paged
 *   with quantisation: element x of head g of k_new (v_new) is stored as the e4m3 code nearest
 *   to the float32 quotient x / k_scale[g] (x / v_scale[g]); ties go to the even mantissa and
 *   magnitudes past 448 saturate to +-448.  k_new, v_new [B][H_kv][d] are `new_dtype`
 *   (GQA_DTYPE_BF16 or GQA_DTYPE_F32).  Overflow and page errors as the 16-bit calls.
 * gqa_decode_fp8: gqa_decode (window = 0) or gqa_decode_window (window >= 1) over the e4m3
 *   cache: the attention of the dequantised values.  Workspace: gqa_decode_workspace_size(...,
 *   GQA_DTYPE_E4M3).  Accuracy: the scores and the softmax weights enter the tensor cores as
 *   several e4m3 terms (q to its full bfloat16 precision, the weights to ~12 significant
 *   bits), with float32 accumulation.
 * gqa_decode_paged_fp8: the paged decode over e4m3 pools; page_size a multiple of 8 that
 *   divides 256 or is a multiple of 256.
 * Scales must be positive and finite (not checked).  NULL scales give GQA_ERR_NULL.
 */
int gqa_kv_append_fp8(const void *k_new, const void *v_new, gqa_dtype_t new_dtype, void *k_cache,
                      void *v_cache, const float *k_scale, const float *v_scale,
                      int32_t *seq_lens, int B, int H_kv, int d, int L_max, int32_t *status,
                      cudaStream_t stream);
int gqa_kv_append_paged_fp8(const void *k_new, const void *v_new, gqa_dtype_t new_dtype,
                            void *k_pool, void *v_pool, const float *k_scale,
                            const float *v_scale, const int32_t *block_table, int max_pages,
                            int32_t *seq_lens, int B, int H_kv, int d, int page_size,
                            int n_pages, int32_t *status, cudaStream_t stream);
int gqa_decode_fp8(const void *q, const void *k_cache, const void *v_cache, const float *k_scale,
                   const float *v_scale, const int32_t *seq_lens, int B, int H_q, int H_kv, int d,
                   int L_max, int window, float scale, float *out, void *workspace,
                   size_t workspace_bytes, int32_t *status, cudaStream_t stream);
int gqa_decode_paged_fp8(const void *q, const void *k_pool, const void *v_pool,
                         const float *k_scale, const float *v_scale, const int32_t *block_table,
                         int max_pages, const int32_t *seq_lens, int B, int H_q, int H_kv, int d,
                         int page_size, int n_pages, float scale, float *out, void *workspace,
                         size_t workspace_bytes, int32_t *status, cudaStream_t stream);

/*
 * gqa_decode_noalloc: gqa_decode without a caller-provided workspace.  (The pages have no
 * counterpart of this call; it exists for callers, not for the method.)
 *
 * For callers that cannot allocate device memory for the workspace: a plugin inside a host
 * framework that owns every device allocation, or a serving loop that must not call cudaMalloc
 * (it can synchronize the device) and has no buffer of its own to lend.  The workspace is a
 * fixed array of GQA_NOALLOC_SCRATCH_BYTES of device memory inside the library; every GPU that
 * loads the library holds it until the process exits.  Arguments and results are those of
 * gqa_decode; the caller still provides q, the caches, seq_lens and out.
 *
 *   - Sizes whose gqa_decode_workspace_size() exceeds GQA_NOALLOC_SCRATCH_BYTES are refused
 *     with GQA_ERR_SCRATCH_LIMIT before anything runs (use gqa_decode with a workspace).
 *   - Every other host-side check of gqa_decode (pointers, alignment, sizes, element type,
 *     scale, device) also runs before anything is queued on `stream`, with gqa_decode's
 *     return codes.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *     with that device current and caches it; make that first call before any stream capture.
 *   - Each call first clears the array's counters with one cudaMemsetAsync on `stream` (the
 *     zero start gqa_decode requires of a workspace), so a call that timed out leaves no
 *     trace for the next one.
 *   - Every call shares the one array and it keeps the last call's contents.  Two calls that
 *     may overlap on the GPU (different streams, or different host threads without ordering)
 *     race on it and produce wrong results; order them on one stream.
 * No cudaMalloc, cudaFree or other allocating routine is called.
 */
#define GQA_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
int gqa_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *seq_lens, int B, int H_q, int H_kv, int d, int L_max,
                       float scale, gqa_dtype_t dtype, float *out, int32_t *status,
                       cudaStream_t stream);

/* gqa_status_string: a static, human-readable string for a GQA_OK / GQA_ERR_* code. */
const char *gqa_status_string(int code);

/*
 * gqa_set_wait_timeout_ns: time limit of every bounded wait inside the decode kernels, for
 * the calls launched after it (process-wide).  ns = 0 restores the default of 2 s.  A
 * kernel whose wait runs out sets GQA_STATUS_WAIT_TIMEOUT, waits for its own copies and
 * tensor-core work already in flight, frees its tensor memory and returns.  Tests use a
 * tiny limit to exercise that path without faulting the GPU.  Returns GQA_OK.
 */
int gqa_set_wait_timeout_ns(unsigned long long ns);

/*
 * gqa_profile_events: measurement hook (process-wide).  When both events are non-NULL, every
 * later gqa_decode records `before_split` on its stream just before the split-KV kernel and
 * `after_split` just after it, so the caller can time that kernel alone with
 * cudaEventElapsedTime.  Pass NULL, NULL to stop.  The caller owns the events.  Returns GQA_OK.
 */
int gqa_profile_events(cudaEvent_t before_split, cudaEvent_t after_split);

#ifdef __cplusplus
}
#endif

#endif /* GQA_H */
