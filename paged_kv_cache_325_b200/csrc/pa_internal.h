// Internal interfaces between the C-ABI front end (pa_api.cu) and the kernel
// translation units.  Not installed; not part of the ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pa.h"

namespace pa {

// ----------------------------------------------------------------- store --
struct StoreArgs {
    const void *k, *v;
    int64_t k_row_stride, v_row_stride;   // elements
    const int32_t *slot_mapping;
    int32_t num_tokens;
    void *k_cache, *v_cache;
    int64_t num_slots;
    int32_t row_elems;                    // num_kv_heads * head_dim
    int32_t *dev_error;
};
cudaError_t launch_store(const StoreArgs &a, cudaStream_t stream);

// ---------------------------------------------------------------- decode --
constexpr int kDecodeTileTokens = 64;

struct DecodePlan {
    int32_t chunk;       // tokens per split, a multiple of kDecodeTileTokens: the finest split the
                         // planning kernel may choose (exactly this one when fixed)
    int32_t max_splits;  // splits of the longest context at that chunk: the partial slots per (s, h)
    int32_t fixed;       // the caller chose the split count: every pair is cut into chunks of `chunk`
};
DecodePlan plan_decode(int32_t batch, int32_t num_kv_heads, int32_t max_context_len, int32_t num_splits,
                       int32_t num_sms);
// Workspace of a decode call: the planning kernel's item table, then (when a pair can be split, or
// extra_slots partials come from elsewhere) fp32 partials and their log-sum-exps.
struct DecodeWorkspace {
    size_t plan_off, o_off, lse_off, total;   // byte offsets from a 256-byte aligned base
};
size_t decode_plan_bytes(const DecodePlan &plan, int32_t batch, int32_t num_kv_heads);   // multiple of 256
DecodeWorkspace decode_workspace_layout(const DecodePlan &plan, int32_t batch, int32_t num_q_heads,
                                        int32_t num_kv_heads, int32_t head_dim, int32_t extra_slots = 0);
constexpr int32_t kDecodeMaxSplits = 32767;     // split index and KV head share one int of an item
constexpr int32_t kDecodeMaxKvHeads = 65535;
constexpr int32_t kDecodeMaxPairs = 1 << 30;    // batch * num_kv_heads: the planning kernel counts pairs in int

struct DecodeArgs {
    void *out;
    const void *q;
    const int32_t *block_table;
    const int32_t *context_lens;
    int32_t *dev_error;
    void *plan_ws;      // the item table (decode_workspace_layout().plan_off)
    float *part_o;      // [batch, Hq, part_slots, D]
    float *part_lse;    // [batch, Hq, part_slots]
    int32_t bt_stride, batch, num_q_heads, num_kv_heads, group, head_dim;
    int32_t num_blocks, block_size, box_tokens, max_context_len;
    DecodePlan plan;
    float scale_log2;
    // the partials of (sequence s, q-head h) sit at slots [part_base, part_base + splits) of part_slots
    int32_t part_slots, part_base;
    int32_t t_offset;        // the split ranges start at this token (shared-prefix decode: P * block_size)
    int32_t shared_blocks;   // checked mode: block_table[s][0..shared_blocks) must equal row 0's
    // varlen rows (the decode rows of a mixed batch): when set, sequence s is this call's work only if it has
    // one new token (cu_q[s+1] - cu_q[s] == 1); its q / out row is cu_q[s] and its context cu_k[s+1] - cu_k[s]
    // (context_lens unused)
    const int32_t *vl_cu_q, *vl_cu_k;
    // store fused into the decode (pa_store_kv_decode): row s of k_new / v_new is sequence s's new token,
    // written to cache slot new_slots[s] (skipped when < 0); NULL new_slots: no store
    const void *k_new, *v_new;
    int64_t kn_stride, vn_stride;   // elements, multiples of 8
    const int32_t *new_slots;
    void *k_cache, *v_cache;
    int64_t num_slots;
    // set by launch_decode (callers leave it NULL): when pairs have only a few splits, the split kernel merges
    // the partials itself -- a pair's only item folds in the part_base partials, and the CTA that finishes a
    // split pair's last split (counted down in these per-pair counters, after the item table in plan_ws, set
    // by the planning kernel) merges all of them -- and no combine kernel runs
    int32_t *merge_count;
};
cudaError_t launch_decode(const DecodeArgs &a, const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                          cudaStream_t stream);

// --------------------------------------------------------------- prefill --
struct PrefillArgs {
    void *out;
    const void *q;
    const int32_t *cu_q, *cu_k, *block_table;
    int32_t *dev_error;
    int32_t bt_stride, batch, num_q_heads, num_kv_heads, group, head_dim;
    int32_t num_blocks, block_size, box_tokens, max_seqlen_q, max_seqlen_k, causal, total_q;
    int32_t ranks;              // pairs of Q tiles of the longest sequence
    void *workspace;            // unit table + hand-out counter (prefill_workspace_bytes)
    float scale_log2;
    // --- used by the shared-prefix decode (zero / NULL for pa_prefill_varlen) ---
    int32_t single_n_new, single_n_k;   // cu_q == NULL: one sequence with these sizes
    int32_t key_chunk, nchunks;         // non-causal: split the keys into chunks of key_chunk (0: one chunk)
    float *part_o, *part_lse;           // non-NULL: write fp32 partials [row, head, part_slots, D] + lse
    int32_t part_slots, part_base;      // partial slots per (row, head); first slot used by chunk 0
    int32_t skip_single;                // mixed batch: sequences with one new token are the decode's work
    // --- pa_store_kv_prefill_varlen (NULL new_slots otherwise): the new keys come from the new K/V rows
    // (row cu_q[s] + i is key c + i of sequence s), which are also stored to their cache slots ---
    const void *k_new, *v_new;
    int64_t kn_stride, vn_stride;       // elements
    const int32_t *new_slots;           // [total_q]
    void *k_cache, *v_cache;
    int64_t num_slots;
};
size_t prefill_workspace_bytes(int32_t batch, int32_t max_seqlen_q, int32_t group, int32_t num_kv_heads,
                               int32_t nchunks = 1);
constexpr int32_t kPrefillMaxBatch = 6144;   // the planning kernel keeps 2 ints per sequence in shared memory
// tm_kn / tm_vn: maps of the new K/V rows, required when a.new_slots is set (ignored otherwise)
cudaError_t launch_prefill(const PrefillArgs &a, const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                           const CUtensorMap &tm_v, cudaStream_t stream, const CUtensorMap *tm_kn = nullptr,
                           const CUtensorMap *tm_vn = nullptr);

// ------------------------------------------------------------ error text --
// Record the text pa_last_error_detail() returns on this thread.
void set_last_error(pa_status status, const char *detail);

// ------------------------------------------------------------- self-test --
cudaError_t launch_selftest_wait(int32_t *dev_error, int64_t max_polls, cudaStream_t stream);
cudaError_t launch_selftest_exp2(const float *x, float *y_poly, float *y_sfu, int32_t n, cudaStream_t stream);

}  // namespace pa
