/*
 * CPU oracle for the paged-KV hot path.  TEST INFRASTRUCTURE ONLY: the tests,
 * the smoke check and the benchmark's CPU-baseline leg are the only callers.
 * The CUDA library never links, includes or calls anything here, and this file
 * uses nothing from it.
 *
 * Plain, slow, obviously correct loops in double precision.  Every function
 * follows the pages' definition step by step and has no blocking, fusion or
 * reordering beyond it:
 *
 *   slot(s, p) = block_table[s][p / B] * B + p % B
 *       address math of the gather ("PagedAttention 的前向计算实现", gsyq.cn
 *       nano-vLLM article, section 4.1, steps 1-3).
 *   gather(s, n) = rows slot(s, 0) .. slot(s, n-1) of the cache
 *       ("gather_from_blocks" in the paged_attention pseudocode of the same
 *       article, section 5.3).
 *   attend(q, K, V) = softmax(q K^T * scale) V
 *       (the attention formula, "万字深度解析 Nano-vLLM", chenxutan.com,
 *       section 1.2; the scale is passed in, as FlashAttention's softmax_scale
 *       in the nano-vllm walkthrough, xingyun3d.csdn.net, section seven).
 *       The softmax is evaluated as exp(x - max) / sum(exp(x - max)), which is
 *       the same function as exp(x) / sum(exp(x)).
 *   kv_head(h) = h / (Hq / Hkv)
 *       (GQA: each KV head is repeated num_kv_groups times with
 *       repeat_interleave, chenxutan.com article, section 3.2.1).
 *   store: cache row slot_mapping[i] := new row i, skipped when the slot is
 *       negative (nano-vllm walkthrough, section seven: a light kernel writes
 *       this step's K/V into the cache through slot_mapping).
 *   decode(s, h)      = attend(q[s, h], gather(s, context_lens[s]))
 *   prefill(s, i, h)  = attend(q[cu_q[s] + i, h], gather(s, c + i + 1)),
 *       c = n_k - n_new, the number of keys before the first new token
 *       (causal alignment of the new segment to the end of the key range,
 *       nano-vllm walkthrough, sections seven and eight: only the uncached
 *       segment is computed, with causal=True over cu_seqlens_k).
 *
 * bf16 inputs are passed as their 16-bit patterns and widened exactly.
 * Return value of every entry: 0 = ok, negative = an index was out of range
 * (the oracle then leaves the affected outputs as NaN).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_bits_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Physical row of logical position p of a sequence whose block list is bt_row. */
static int64_t slot_of(const int32_t *bt_row, int64_t p, int32_t block_size) {
    return (int64_t)bt_row[p / block_size] * block_size + p % block_size;
}

/*
 * Gather n rows of one KV head of one sequence into dst[n][D] (double).
 * Returns -1 if a block id is outside [0, num_blocks).
 */
static int gather(double *dst, const uint16_t *cache, const int32_t *bt_row, int64_t n,
                  int32_t block_size, int32_t num_blocks, int32_t num_kv_heads, int32_t kv_head,
                  int32_t head_dim) {
    for (int64_t p = 0; p < n; ++p) {
        int32_t blk = bt_row[p / block_size];
        if (blk < 0 || blk >= num_blocks) return -1;
        int64_t slot = slot_of(bt_row, p, block_size);
        const uint16_t *row = cache + (slot * num_kv_heads + kv_head) * (int64_t)head_dim;
        for (int32_t d = 0; d < head_dim; ++d) dst[p * head_dim + d] = bf16_bits_to_double(row[d]);
    }
    return 0;
}

/* out[D] = softmax_j(scale * q . K_j) weighted sum of V_j, j = 0..n-1. */
static void attend(double *out, const double *q, const double *K, const double *V, int64_t n,
                   int32_t head_dim, double scale, double *score) {
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j) {
        double dot = 0.0;
        for (int32_t d = 0; d < head_dim; ++d) dot += q[d] * K[j * head_dim + d];
        score[j] = scale * dot;
        if (score[j] > m) m = score[j];
    }
    double z = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        score[j] = exp(score[j] - m);
        z += score[j];
    }
    for (int32_t d = 0; d < head_dim; ++d) {
        double acc = 0.0;
        for (int64_t j = 0; j < n; ++j) acc += score[j] * V[j * head_dim + d];
        out[d] = acc / z;
    }
}

static void fill_nan(double *out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = NAN;
}

/* ------------------------------------------------------------------------- */

int oracle_store(const uint16_t *k, const uint16_t *v, int64_t k_row_stride, int64_t v_row_stride,
                 const int32_t *slot_mapping, int32_t num_tokens, uint16_t *k_cache, uint16_t *v_cache,
                 int64_t num_slots, int32_t num_kv_heads, int32_t head_dim) {
    int64_t row = (int64_t)num_kv_heads * head_dim;
    int rc = 0;
    for (int32_t i = 0; i < num_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0) continue;
        if (slot >= num_slots) { rc = -1; continue; }
        memcpy(k_cache + slot * row, k + (int64_t)i * k_row_stride, (size_t)row * 2);
        memcpy(v_cache + slot * row, v + (int64_t)i * v_row_stride, (size_t)row * 2);
    }
    return rc;
}

/*
 * Decode for a list of (sequence, q-head) pairs: out[r][D] for pair r.
 * All pairs when seq_idx == NULL (then nrows = batch * Hq, r = s * Hq + h).
 */
int oracle_decode(double *out, int32_t nrows, const int32_t *seq_idx, const int32_t *head_idx,
                  const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                  const int32_t *block_table, int32_t block_table_stride, const int32_t *context_lens,
                  int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                  int32_t num_blocks, int32_t block_size, double scale) {
    int32_t group = num_q_heads / num_kv_heads;
    int rc = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(min : rc)
    for (int32_t r = 0; r < nrows; ++r) {
        int32_t s = seq_idx ? seq_idx[r] : r / num_q_heads;
        int32_t h = head_idx ? head_idx[r] : r % num_q_heads;
        double *o = out + (int64_t)r * head_dim;
        int64_t n = (s >= 0 && s < batch) ? context_lens[s] : -1;
        if (n < 1 || n > (int64_t)block_table_stride * block_size || h < 0 || h >= num_q_heads) {
            fill_nan(o, head_dim);
            rc = -1;
            continue;
        }
        double *K = malloc(sizeof(double) * n * head_dim);
        double *V = malloc(sizeof(double) * n * head_dim);
        double *sc = malloc(sizeof(double) * n);
        double qd[256];
        const int32_t *bt = block_table + (int64_t)s * block_table_stride;
        int32_t kvh = h / group;
        if (gather(K, k_cache, bt, n, block_size, num_blocks, num_kv_heads, kvh, head_dim) ||
            gather(V, v_cache, bt, n, block_size, num_blocks, num_kv_heads, kvh, head_dim)) {
            fill_nan(o, head_dim);
            rc = -1;
        } else {
            const uint16_t *qr = q + ((int64_t)s * num_q_heads + h) * head_dim;
            for (int32_t d = 0; d < head_dim; ++d) qd[d] = bf16_bits_to_double(qr[d]);
            attend(o, qd, K, V, n, head_dim, scale, sc);
        }
        free(K);
        free(V);
        free(sc);
    }
    return rc;
}

/*
 * Varlen prefill for a list of (query token, q-head) pairs: out[r][D].
 * All rows when tok_idx == NULL (then nrows = total_q * Hq, r = t * Hq + h).
 * Query token t belongs to the sequence s with cu_q[s] <= t < cu_q[s+1].
 */
int oracle_prefill(double *out, int32_t nrows, const int32_t *tok_idx, const int32_t *head_idx,
                   const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                   const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, const int32_t *block_table,
                   int32_t block_table_stride, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                   int32_t head_dim, int32_t num_blocks, int32_t block_size, double scale, int32_t causal) {
    int32_t group = num_q_heads / num_kv_heads;
    int rc = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(min : rc)
    for (int32_t r = 0; r < nrows; ++r) {
        int32_t t = tok_idx ? tok_idx[r] : r / num_q_heads;
        int32_t h = head_idx ? head_idx[r] : r % num_q_heads;
        double *o = out + (int64_t)r * head_dim;
        int32_t s = -1;
        for (int32_t b = 0; b < batch; ++b)
            if (cu_seqlens_q[b] <= t && t < cu_seqlens_q[b + 1]) { s = b; break; }
        if (s < 0 || h < 0 || h >= num_q_heads) { fill_nan(o, head_dim); rc = -1; continue; }
        int64_t n_new = cu_seqlens_q[s + 1] - cu_seqlens_q[s];
        int64_t n_k = cu_seqlens_k[s + 1] - cu_seqlens_k[s];
        int64_t c = n_k - n_new;
        int64_t i = t - cu_seqlens_q[s];
        int64_t n = causal ? c + i + 1 : n_k;
        if (c < 0 || n < 1 || n_k > (int64_t)block_table_stride * block_size) {
            fill_nan(o, head_dim);
            rc = -1;
            continue;
        }
        double *K = malloc(sizeof(double) * n * head_dim);
        double *V = malloc(sizeof(double) * n * head_dim);
        double *sc = malloc(sizeof(double) * n);
        double qd[256];
        const int32_t *bt = block_table + (int64_t)s * block_table_stride;
        int32_t kvh = h / group;
        if (gather(K, k_cache, bt, n, block_size, num_blocks, num_kv_heads, kvh, head_dim) ||
            gather(V, v_cache, bt, n, block_size, num_blocks, num_kv_heads, kvh, head_dim)) {
            fill_nan(o, head_dim);
            rc = -1;
        } else {
            const uint16_t *qr = q + ((int64_t)t * num_q_heads + h) * head_dim;
            for (int32_t d = 0; d < head_dim; ++d) qd[d] = bf16_bits_to_double(qr[d]);
            attend(o, qd, K, V, n, head_dim, scale, sc);
        }
        free(K);
        free(V);
        free(sc);
    }
    return rc;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
