/*
 * pa.h -- C ABI of the B200 (sm_100a) paged-KV attention library (libpagedattn.so).
 *
 * Three operations make up one attention layer call of a paged-KV inference
 * engine of the nano-vllm kind:
 *
 *   pa_store_kv        write this step's new K/V rows into the block-paged cache
 *   pa_decode          one query token per sequence attends to its whole context
 *   pa_prefill_varlen  the new (uncached) tokens of each prompt attend causally
 *                      to the cached prefix plus themselves
 *
 * The call order follows the attention forward of the nano-vllm walkthrough
 * (xingyun3d.csdn.net, section seven "后端执行（cuda 算子）"): store first, then
 * prefill or decode on the same stream.  Argument names follow the per-step
 * context object of the same page (section eight "序列与上下文"): slot_mapping,
 * context_lens, block_tables, cu_seqlens_q/k, max_seqlen_q/k.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE memory owned by the caller.  The library
 *    never allocates, frees or retains them and keeps no state between calls
 *    other than a per-device cache of kernel attributes.
 *  - Element type: K, V, Q and outputs are bfloat16 (passed as void*); every
 *    index array is int32.
 *  - Cache layout: k_cache and v_cache are [num_blocks, block_size,
 *    num_kv_heads, head_dim], contiguous, 16-byte aligned.  Token p of a
 *    sequence lives in slot block_table[s][p / block_size] * block_size +
 *    p % block_size (block index and in-block offset, gsyq.cn nano-vLLM
 *    article, section 4.1).
 *  - Supported shapes: head_dim in {64, 128}; block_size a power of two in
 *    [16, 256]; num_q_heads a multiple of num_kv_heads with
 *    num_q_heads / num_kv_heads <= 16.  Anything else returns
 *    PA_ERR_UNSUPPORTED.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *    entry point is asynchronous: it validates its host-side arguments
 *    synchronously, enqueues its kernels and returns.
 *  - Host-side errors (bad scalars, null or misaligned pointers, a workspace
 *    that is too small) return an error status before anything is enqueued.
 *    A failed launch returns PA_ERR_CUDA.  pa_last_error_detail() gives a
 *    human-readable reason for the last error on the calling thread.
 *  - Checked mode: when `dev_error` is non-NULL (device memory, one int32
 *    the caller zeroes), kernels validate device-resident indices and OR one
 *    of the PA_DEVERR_* bits into it instead of reading or writing out of
 *    range; the affected outputs are left unspecified.  Kernels never trap.
 *    With dev_error == NULL the same checks run but nothing is reported:
 *    cache accesses stay inside the cache either way (stores skip slots past
 *    its end; reads go through TMA tensor maps, which zero-fill out-of-range
 *    coordinates).
 */
#ifndef PAGED_KV_PA_H
#define PAGED_KV_PA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,   /* a pointer is NULL or misaligned, a size is negative, ...   */
    PA_ERR_UNSUPPORTED = 2,   /* a valid shape this build has no kernel for                 */
    PA_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed (launch, attribute, ...) */
    PA_ERR_DEVICE_CHECK = 4,  /* a checked-mode kernel found a bad index (see PA_DEVERR_*)  */
    PA_ERR_TIMEOUT = 5,       /* a bounded device-side wait ran out                         */
    PA_ERR_WORKSPACE = 6      /* the workspace is NULL or smaller than the size query says  */
} pa_status;

/* Bits a kernel ORs into *dev_error in checked mode. */
#define PA_DEVERR_BLOCK_ID    0x1  /* a block_table entry that a context needs is outside [0, num_blocks) */
#define PA_DEVERR_SLOT        0x2  /* a slot_mapping entry is >= num_blocks * block_size                 */
#define PA_DEVERR_CONTEXT_LEN 0x4  /* context_lens[s] < 1, > max_context_len or > table capacity         */
#define PA_DEVERR_SEQLENS     0x8  /* cu_seqlens not monotone, n_new > n_k, or a length > max_seqlen     */
#define PA_DEVERR_TIMEOUT     0x10 /* a bounded mbarrier wait gave up                                     */

/* Static string naming a status code. */
PA_API const char *pa_status_string(int status);

/* Text describing the last error returned on the calling thread ("" if none). */
PA_API const char *pa_last_error_detail(void);

/* Library ABI version (major * 100 + minor). */
PA_API int pa_version(void);

/*
 * pa_store_kv -- store_kvcache.
 *
 * For every i in [0, num_tokens) with slot_mapping[i] >= 0:
 *     k_cache.view(num_blocks * block_size, num_kv_heads, head_dim)[slot_mapping[i]] = k[i]
 *     v_cache.view(...)[slot_mapping[i]]                                          = v[i]
 * a bit-exact copy ("a light kernel writes this step's K/V into the
 * pre-allocated cache through slot_mapping", nano-vllm walkthrough, section
 * seven; the Triton store kernel of the gitcode.csdn.net nano-vLLM article,
 * section 3.4).  Negative slots are skipped (padding rows).  Two rows that
 * name the same slot in one call race: the caller must not pass duplicates.
 *
 *   k, v           [num_tokens, num_kv_heads, head_dim] bf16; row i starts at
 *                  element i * k_row_stride (resp. v_row_stride); each row's
 *                  num_kv_heads * head_dim elements are contiguous.
 *   slot_mapping   [num_tokens] int32, device.
 *   k_cache/v_cache  the paged cache (written in place).
 * num_tokens == 0 is a no-op that returns PA_OK.
 */
PA_API pa_status pa_store_kv(const void *k, const void *v, int64_t k_row_stride, int64_t v_row_stride,
                      const int32_t *slot_mapping, int32_t num_tokens, void *k_cache, void *v_cache,
                      int32_t num_blocks, int32_t block_size, int32_t num_kv_heads, int32_t head_dim,
                      int32_t *dev_error, void *stream);

/*
 * Bytes of device workspace pa_decode needs for these sizes on the current
 * device (0 only when batch <= 0): the planning kernel's table of work items,
 * a counter per (sequence, KV head) and, when a context may be split, the
 * per-split partial results.
 */
PA_API size_t pa_decode_workspace_size(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                int32_t max_context_len, int32_t block_size);

/*
 * pa_decode -- paged decode attention (the flash_attn_with_kvcache call with
 * cache_seqlens = context_lens and block_table, nano-vllm walkthrough,
 * section seven).  For every sequence s and q-head h:
 *
 *   out[s, h] = sum_j softmax_j(softmax_scale * q[s, h] . K_j) V_j,
 *               j over the context_lens[s] tokens of sequence s,
 *
 * the attention formula of the chenxutan.com article (section 1.2), with K_j,
 * V_j of KV head h / (num_q_heads / num_kv_heads) (GQA repeat_interleave,
 * same article, section 3.2.1) gathered through block_table (the gather of the
 * gsyq.cn article, sections 4.1 and 5.3).  context_lens counts the token
 * stored by this step's pa_store_kv.
 *
 *   out, q           [batch, num_q_heads, head_dim] bf16, contiguous.
 *   block_table      [batch, block_table_stride] int32; entries past
 *                    ceil(context_lens[s] / block_size) are never read.
 *   context_lens     [batch] int32, each in [1, max_context_len].
 *   max_context_len  host-side upper bound of context_lens (sizes the split).
 *   workspace        device scratch of at least pa_decode_workspace_size()
 *                    bytes, 256-byte aligned.  Its contents need no
 *                    initialisation and are garbage afterwards.  Two calls
 *                    whose kernels may overlap on the GPU need two workspaces.
 *
 * Two or three kernels on `stream`: a one-CTA planning kernel reads
 * context_lens and writes a table of work items (a whole (sequence, KV head),
 * or one split of a context far longer than the average per-CTA load): the
 * first split of pair c for decode CTA c, which starts on it before the table
 * exists, then the rest longest first; the persistent decode kernel takes
 * items with an atomic counter.  Partial results of split contexts are merged
 * by log-sum-exp: inside the decode kernel, by the CTA that finishes a pair's
 * last split, when the plan allows at most 8 splits per pair; otherwise by a
 * third, combine kernel.
 */
PA_API pa_status pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *block_table, int32_t block_table_stride, const int32_t *context_lens,
                    int32_t batch, int32_t max_context_len, int32_t num_q_heads, int32_t num_kv_heads,
                    int32_t head_dim, int32_t num_blocks, int32_t block_size, float softmax_scale,
                    void *workspace, size_t workspace_bytes, int32_t *dev_error, void *stream);

/*
 * pa_store_kv_decode -- pa_store_kv followed by pa_decode, in one kernel launch
 * (the decode step of the walkthrough, section seven: store_kvcache of this
 * step's K/V through slot_mapping, then flash_attn_with_kvcache).  Row s of
 * k / v is the new token of sequence s (num_tokens == batch), stored at slot
 * slot_mapping[s]; context_lens[s] counts it, as in pa_decode.  Results are
 * those of pa_store_kv then pa_decode on the same stream: the cache holds the
 * new rows afterwards, bit for bit, and out is the decode of the updated cache.
 *
 * The new token of sequence s is the one at position context_lens[s] - 1, so
 * slot_mapping[s] must be either negative (a padding row: nothing is stored and
 * the decode reads the cache as it is) or that position's slot,
 * block_table[s][(context_lens[s]-1) / block_size] * block_size
 * + (context_lens[s]-1) % block_size.  A different slot is still written, but
 * the decode does not see the new row there; checked mode reports it as
 * PA_DEVERR_SLOT, as it does a slot >= num_blocks * block_size (not written).
 * A row of a sequence whose context length is rejected (below 1, above
 * max_context_len or past its block_table row; checked mode reports
 * PA_DEVERR_CONTEXT_LEN) is still stored, as pa_store_kv would store it; only
 * that sequence's decode is skipped and its output rows are left untouched.
 *
 *   k, v          [batch, num_kv_heads, head_dim] bf16, row s at element
 *                 s * k_row_stride (v_row_stride); the rows must be 16-byte
 *                 aligned (strides a multiple of 8 elements), otherwise
 *                 PA_ERR_UNSUPPORTED: use pa_store_kv + pa_decode.
 *   slot_mapping  [batch] int32, device.
 *   everything else as pa_decode, with the same workspace size
 *   (pa_decode_workspace_size).
 */
PA_API pa_status pa_store_kv_decode(const void *k, const void *v, int64_t k_row_stride, int64_t v_row_stride,
                                    const int32_t *slot_mapping, void *out, const void *q, void *k_cache,
                                    void *v_cache, const int32_t *block_table, int32_t block_table_stride,
                                    const int32_t *context_lens, int32_t batch, int32_t max_context_len,
                                    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                    int32_t num_blocks, int32_t block_size, float softmax_scale, void *workspace,
                                    size_t workspace_bytes, int32_t *dev_error, void *stream);

/*
 * pa_decode_split -- pa_decode with the number of context splits chosen by
 * the caller (num_splits > 0), like FlashAttention's num_splits argument;
 * num_splits == 0 picks the split automatically, exactly as pa_decode does.
 * The context is cut into splits of ceil(max_context_len / num_splits)
 * tokens rounded up to a multiple of 64.  The result is the same function
 * either way; only the rounding order of the fp32 accumulation changes.
 * Workspace: pa_decode_split_workspace_size() with the same num_splits.
 */
PA_API size_t pa_decode_split_workspace_size(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                      int32_t max_context_len, int32_t num_splits);
PA_API pa_status pa_decode_split(void *out, const void *q, const void *k_cache, const void *v_cache,
                          const int32_t *block_table, int32_t block_table_stride, const int32_t *context_lens,
                          int32_t batch, int32_t max_context_len, int32_t num_q_heads, int32_t num_kv_heads,
                          int32_t head_dim, int32_t num_blocks, int32_t block_size, float softmax_scale,
                          int32_t num_splits, void *workspace, size_t workspace_bytes, int32_t *dev_error,
                          void *stream);

/*
 * pa_decode_shared_prefix -- pa_decode for a batch whose sequences all start
 * with the same num_shared_blocks physical blocks (a prefix-cache hit shared by
 * the whole batch: block_table[s][0 .. num_shared_blocks) is the same for every
 * s, as the BlockManager's whole-block prefix hashing produces, nano-vllm
 * walkthrough, section five).  It computes exactly what pa_decode computes, but
 * reads the shared blocks once per KV head instead of once per sequence:
 *   1. all batch x G query rows of a KV head attend to the shared keys
 *      together on the tensor cores (non-causal, the keys cut into chunks),
 *      each chunk giving an fp32 partial and its log-sum-exp;
 *   2. the split-KV decode covers each sequence's private tokens
 *      [num_shared_blocks * block_size, context_lens[s]);
 *   3. all partials of a (sequence, q-head) are merged by log-sum-exp (in the
 *      decode kernel when its plan gives at most 8 splits per pair, else by a
 *      combine kernel; a sequence with no private token by the planning
 *      kernel).
 * Every context_lens[s] must be >= num_shared_blocks * block_size (checked
 * mode reports PA_DEVERR_CONTEXT_LEN; a table row whose first blocks differ
 * from row 0's is reported as PA_DEVERR_BLOCK_ID).  The GQA group must divide
 * 128.  Workspace: pa_decode_shared_prefix_workspace_size() bytes, 256-byte
 * aligned, no initialisation needed.
 */
PA_API size_t pa_decode_shared_prefix_workspace_size(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                                     int32_t head_dim, int32_t max_context_len, int32_t block_size,
                                                     int32_t num_shared_blocks);
PA_API pa_status pa_decode_shared_prefix(void *out, const void *q, const void *k_cache, const void *v_cache,
                                         const int32_t *block_table, int32_t block_table_stride,
                                         const int32_t *context_lens, int32_t batch, int32_t max_context_len,
                                         int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                         int32_t num_blocks, int32_t block_size, float softmax_scale,
                                         int32_t num_shared_blocks, void *workspace, size_t workspace_bytes,
                                         int32_t *dev_error, void *stream);

/*
 * pa_decode_noalloc -- pa_decode for callers that cannot allocate device
 * memory (no counterpart in the pages: it exists for integration, not for the
 * method).  Some hosts own every device allocation themselves -- a plugin
 * runtime, or an engine that gives all spare HBM to its KV-cache pool -- and
 * cannot hand this library a workspace.  This variant computes exactly what
 * pa_decode computes, but takes its split scratch from a fixed array compiled
 * into the library: pa_decode_noalloc_max_scratch_bytes() bytes (8 MiB) per
 * GPU, held by every GPU that loads the library until the process exits.  It
 * calls no cudaMalloc, cudaFree or other allocating routine.
 *
 * Arguments are those of pa_decode without the workspace.  Sizes whose split
 * scratch (pa_decode_workspace_size) exceeds the array are rejected with
 * PA_ERR_WORKSPACE before anything is enqueued.  Every call looks up the
 * array's address in the current device's context (cudaGetSymbolAddress) and
 * keeps nothing, so the call stays correct after the context is torn down and
 * created again (cudaDeviceReset); the first call on a device may load the
 * library's device code, so make it before any stream capture.
 * Every call on a device shares the one array and it keeps the last call's
 * contents; nothing in it has to start at zero (each call writes every
 * partial it reads).  Calls whose kernels overlap on the GPU -- on different
 * streams, or concurrently from several host threads -- race on the array:
 * serialise them (one stream, or events).
 */
PA_API size_t pa_decode_noalloc_max_scratch_bytes(void);
PA_API pa_status pa_decode_noalloc(void *out, const void *q, const void *k_cache, const void *v_cache,
                                   const int32_t *block_table, int32_t block_table_stride,
                                   const int32_t *context_lens, int32_t batch, int32_t max_context_len,
                                   int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks,
                                   int32_t block_size, float softmax_scale, int32_t *dev_error, void *stream);

/*
 * Bytes of device workspace pa_prefill_varlen needs: a table of the work units
 * (pairs of 128-row Q tiles), ordered from the most to the least expensive,
 * and the counter the persistent kernel hands them out with.  It grows with
 * batch and max_seqlen_q (a few KB for a dozen prompts of 2k tokens).
 */
PA_API size_t pa_prefill_workspace_size(int32_t batch, int32_t max_seqlen_q, int32_t num_q_heads,
                                 int32_t num_kv_heads, int32_t head_dim);

/*
 * pa_prefill_varlen -- varlen causal prefill over the paged cache (the
 * flash_attn_varlen_func call with cu_seqlens_q/k, max_seqlen_q/k,
 * causal=True and block_table, nano-vllm walkthrough, section seven).
 *
 * Sequence s has n_new = cu_seqlens_q[s+1] - cu_seqlens_q[s] query tokens and
 * n_k = cu_seqlens_k[s+1] - cu_seqlens_k[s] keys; the first c = n_k - n_new
 * keys are a cached prefix (a prefix-cache hit) and the last n_new keys are
 * the query tokens themselves, already stored by pa_store_kv.  New token i
 * sits at absolute position c + i and, with causal != 0, attends to keys
 * 0 .. c + i (all n_k keys when causal == 0):
 *
 *   out[cu_q[s] + i, h] = sum_j softmax_j(softmax_scale * q[cu_q[s] + i, h] . K_j) V_j
 *
 *   out, q           [total_q, num_q_heads, head_dim] bf16, contiguous;
 *                    total_q (host) is their row count, >= cu_seqlens_q[batch]
 *                    (checked mode reports a sequence that ends past it, and
 *                    no row past it is ever read or written).
 *   cu_seqlens_q/k   [batch + 1] int32, device, starting at 0.
 *   max_seqlen_q/k   host-side upper bounds of n_new and n_k.
 *   block_table      [batch, block_table_stride] int32.
 *   workspace        device scratch of at least pa_prefill_workspace_size()
 *                    bytes, 256-byte aligned; no initialisation needed (a
 *                    planning kernel on the same stream rewrites it every call),
 *                    garbage afterwards.  batch <= 6144.
 *
 * Two kernels run: a one-CTA planning kernel that validates every sequence and
 * orders the work units, then the persistent prefill kernel (launched with
 * programmatic dependent launch so its prologue overlaps the planning).
 */
PA_API pa_status pa_prefill_varlen(void *out, const void *q, int32_t total_q, const void *k_cache, const void *v_cache,
                            const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, int32_t max_seqlen_q,
                            int32_t max_seqlen_k, const int32_t *block_table, int32_t block_table_stride,
                            int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                            int32_t num_blocks, int32_t block_size, float softmax_scale, int32_t causal,
                            void *workspace, size_t workspace_bytes, int32_t *dev_error, void *stream);

/*
 * pa_prefill_varlen_mixed -- pa_prefill_varlen for a batch that mixes prompts
 * with decode steps (the pages' per-step context carries both cu_seqlens_q/k
 * and context_lens; nano-vllm walkthrough, section eight).  Sequences with
 * exactly one new token are computed by the split-KV decode kernel (their q /
 * out row is cu_seqlens_q[s], their context n_k), the others by the prefill
 * kernel, both in this call and on `stream`.  The result is the function
 * pa_prefill_varlen computes (causal); only the kernels differ: a one-token
 * row in the prefill kernel costs a 128-row tile of the tensor cores, in the
 * decode kernel one pass over its keys.  Arguments as pa_prefill_varlen
 * (always causal); workspace: pa_prefill_varlen_mixed_workspace_size() bytes,
 * 256-byte aligned, no initialisation needed.
 */
PA_API size_t pa_prefill_varlen_mixed_workspace_size(int32_t batch, int32_t max_seqlen_q, int32_t max_seqlen_k,
                                                     int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim);
PA_API pa_status pa_prefill_varlen_mixed(void *out, const void *q, int32_t total_q, const void *k_cache,
                                         const void *v_cache, const int32_t *cu_seqlens_q,
                                         const int32_t *cu_seqlens_k, int32_t max_seqlen_q, int32_t max_seqlen_k,
                                         const int32_t *block_table, int32_t block_table_stride, int32_t batch,
                                         int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                         int32_t num_blocks, int32_t block_size, float softmax_scale,
                                         void *workspace, size_t workspace_bytes, int32_t *dev_error, void *stream);

/*
 * pa_store_kv_prefill_varlen -- pa_store_kv of the prompts' new K/V rows
 * followed by pa_prefill_varlen, in one launch, with the new keys read
 * straight from the new K/V rows instead of back from the cache (the prefill
 * step of the walkthrough, section seven: store_kvcache through slot_mapping,
 * then flash_attn_varlen_func over the paged cache).  Row cu_seqlens_q[s] + i
 * of k / v (and of slot_mapping) is sequence s's new token at position c + i,
 * c = n_k - n_new the cached prefix (whole blocks).  Results are those of
 * pa_store_kv then pa_prefill_varlen on the same stream: the cache holds the
 * new rows afterwards, bit for bit, and out is the prefill of the updated
 * cache -- provided each slot_mapping row is the slot that block_table gives
 * for that token's position, which checked mode verifies (PA_DEVERR_SLOT; a
 * negative slot is also reported, and not stored, while the prefill still uses
 * the row).  No other kernel of the launch reads the stored slots.
 *
 *   k, v          [total_q, num_kv_heads, head_dim] bf16, row t at element
 *                 t * k_row_stride (v_row_stride); 16-byte aligned rows
 *                 (strides a multiple of 8 elements), otherwise
 *                 PA_ERR_UNSUPPORTED: use pa_store_kv + pa_prefill_varlen.
 *   slot_mapping  [total_q] int32, device.
 *   everything else as pa_prefill_varlen (same workspace size).
 */
PA_API pa_status pa_store_kv_prefill_varlen(const void *k, const void *v, int64_t k_row_stride, int64_t v_row_stride,
                                            const int32_t *slot_mapping, void *out, const void *q, int32_t total_q,
                                            void *k_cache, void *v_cache, const int32_t *cu_seqlens_q,
                                            const int32_t *cu_seqlens_k, int32_t max_seqlen_q, int32_t max_seqlen_k,
                                            const int32_t *block_table, int32_t block_table_stride, int32_t batch,
                                            int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                            int32_t num_blocks, int32_t block_size, float softmax_scale,
                                            int32_t causal, void *workspace, size_t workspace_bytes,
                                            int32_t *dev_error, void *stream);

/*
 * pa_selftest_bounded_wait -- exercises the library's bounded mbarrier wait:
 * one CTA waits for an arrival that never comes, gives up after
 * `max_polls` polls, ORs PA_DEVERR_TIMEOUT into *dev_error and exits
 * normally, so the context stays usable.  Used by the tests of the timeout
 * path; has no counterpart in the attention method itself.
 */
PA_API pa_status pa_selftest_bounded_wait(int32_t *dev_error, int64_t max_polls, void *stream);

/*
 * pa_selftest_exp2 -- evaluates, for each x[i] (device float array of n
 * values), the two ways the prefill softmax computes 2^x: y_poly[i] from the
 * library's own polynomial on the FMA pipe (round-to-nearest range reduction
 * and a degree-3 fit of 2^f on [-1/2, 1/2], relative error below 1e-4; inputs
 * below -125 give 2^-125) and y_sfu[i] from the special-function unit's
 * ex2.approx.  All three arrays are caller-owned device memory.  Used by the
 * tests to hold the polynomial to its error bound; has no counterpart in the
 * attention method itself.  Errors: PA_ERR_INVALID_ARG for n < 0 or NULL /
 * misaligned arrays.
 */
PA_API pa_status pa_selftest_exp2(const float *x, float *y_poly, float *y_sfu, int32_t n, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_KV_PA_H */
