// C-ABI front end of libpagedattn.so: host-side validation, TMA tensor-map
// encoding and dispatch to the kernels.  Every entry point is declared and
// documented in include/pa.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <string>

#include "pa.h"
#include "pa_internal.h"

namespace {

thread_local std::string g_last_error;

pa_status fail(pa_status st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
pa_status fail(pa_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

pa_status ok() {
    g_last_error.clear();
    return PA_OK;
}

pa_status cuda_fail(cudaError_t e, const char *what) {
    return fail(PA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool pow2(int32_t x) { return x > 0 && (x & (x - 1)) == 0; }

// cuTensorMapEncodeTiled from the driver, looked up at first use so that the
// library loads (and its host-side checks run) on machines without a driver.
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

int num_sms_current() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

// A [rows, heads, head_dim] bf16 tensor viewed in 3-D for TMA: dims (innermost
// first) {head_dim, heads, rows}, box {64, box_heads, box_rows}, 128-byte
// swizzle (each box row of 64 bf16 values is one 128-byte swizzle row).
pa_status encode_rows(CUtensorMap *map, const void *base, int64_t rows, int32_t heads, int32_t head_dim,
                      int32_t box_heads, int32_t box_rows, int64_t row_stride = 0) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable (no CUDA driver?)");
    cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)heads, (cuuint64_t)rows};
    // row_stride (elements; 0: heads * head_dim) must be a multiple of 8 (the 16-byte stride rule)
    const int64_t rs = row_stride > 0 ? row_stride : (int64_t)heads * head_dim;
    cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2, (cuuint64_t)rs * 2};
    cuuint32_t box[3] = {64u, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
    return PA_OK;
}

pa_status check_cache_shape(int32_t num_blocks, int32_t block_size, int32_t num_kv_heads, int32_t head_dim) {
    if (num_blocks < 1 || num_kv_heads < 1) return fail(PA_ERR_INVALID_ARG, "num_blocks and num_kv_heads must be >= 1");
    if (head_dim != 64 && head_dim != 128) return fail(PA_ERR_UNSUPPORTED, "head_dim %d not in {64, 128}", head_dim);
    if (!pow2(block_size) || block_size < 16 || block_size > 256)
        return fail(PA_ERR_UNSUPPORTED, "block_size %d is not a power of two in [16, 256]", block_size);
    if ((int64_t)num_blocks * block_size >= (int64_t(1) << 31))
        return fail(PA_ERR_UNSUPPORTED, "num_blocks * block_size must be < 2^31");
    return PA_OK;
}

pa_status check_heads(int32_t num_q_heads, int32_t num_kv_heads) {
    if (num_q_heads < 1 || num_kv_heads < 1) return fail(PA_ERR_INVALID_ARG, "head counts must be >= 1");
    if (num_q_heads % num_kv_heads != 0)
        return fail(PA_ERR_INVALID_ARG, "num_q_heads %d is not a multiple of num_kv_heads %d", num_q_heads,
                    num_kv_heads);
    if (num_q_heads / num_kv_heads > 16)
        return fail(PA_ERR_UNSUPPORTED, "GQA group %d > 16", num_q_heads / num_kv_heads);
    return PA_OK;
}

}  // namespace

namespace pa {
void set_last_error(pa_status status, const char *detail) { fail(status, "%s", detail); }
}  // namespace pa

extern "C" {

const char *pa_status_string(int status) {
    switch (status) {
        case PA_OK: return "PA_OK";
        case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
        case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
        case PA_ERR_CUDA: return "PA_ERR_CUDA";
        case PA_ERR_DEVICE_CHECK: return "PA_ERR_DEVICE_CHECK";
        case PA_ERR_TIMEOUT: return "PA_ERR_TIMEOUT";
        case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE";
        default: return "PA_ERR_UNKNOWN";
    }
}

const char *pa_last_error_detail(void) { return g_last_error.c_str(); }

int pa_version(void) { return 100; }

pa_status pa_store_kv(const void *k, const void *v, int64_t k_row_stride, int64_t v_row_stride,
                      const int32_t *slot_mapping, int32_t num_tokens, void *k_cache, void *v_cache,
                      int32_t num_blocks, int32_t block_size, int32_t num_kv_heads, int32_t head_dim,
                      int32_t *dev_error, void *stream) {
    if (num_tokens < 0) return fail(PA_ERR_INVALID_ARG, "num_tokens < 0");
    pa_status st = check_cache_shape(num_blocks, block_size, num_kv_heads, head_dim);
    if (st != PA_OK) return st;
    const int64_t row = (int64_t)num_kv_heads * head_dim;
    if (k_row_stride < row || v_row_stride < row)
        return fail(PA_ERR_INVALID_ARG, "row strides must be >= num_kv_heads * head_dim");
    if (num_tokens == 0) return ok();
    if (!k || !v || !slot_mapping || !k_cache || !v_cache) return fail(PA_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned(k, 2) || !aligned(v, 2) || !aligned(slot_mapping, 4) || !aligned(k_cache, 16) ||
        !aligned(v_cache, 16) || (dev_error && !aligned(dev_error, 4)))
        return fail(PA_ERR_INVALID_ARG, "misaligned pointer");
    pa::StoreArgs a;
    a.k = k;
    a.v = v;
    a.k_row_stride = k_row_stride;
    a.v_row_stride = v_row_stride;
    a.slot_mapping = slot_mapping;
    a.num_tokens = num_tokens;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.num_slots = (int64_t)num_blocks * block_size;
    a.row_elems = (int32_t)row;
    a.dev_error = dev_error;
    cudaError_t e = pa::launch_store(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "store kernel launch");
    return ok();
}

size_t pa_decode_workspace_size(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                int32_t max_context_len, int32_t block_size) {
    (void)block_size;
    if (batch <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || max_context_len <= 0) return 0;
    pa::DecodePlan plan = pa::plan_decode(batch, num_kv_heads, max_context_len, 0, num_sms_current());
    return pa::decode_workspace_layout(plan, batch, num_q_heads, num_kv_heads, head_dim).total;
}

// The new token rows of pa_store_kv_decode (NULL for the plain decode).
struct FusedStore {
    const void *k, *v;
    int64_t k_row_stride, v_row_stride;
    const int32_t *slot_mapping;
};

static pa_status decode_impl(void *out, const void *q, const void *k_cache, const void *v_cache,
                             const int32_t *block_table, int32_t block_table_stride, const int32_t *context_lens,
                             int32_t batch, int32_t max_context_len, int32_t num_q_heads, int32_t num_kv_heads,
                             int32_t head_dim, int32_t num_blocks, int32_t block_size, float softmax_scale,
                             int32_t num_splits, void *workspace, size_t workspace_bytes, int32_t *dev_error,
                             void *stream, const FusedStore *fs = nullptr) {
    if (batch < 0) return fail(PA_ERR_INVALID_ARG, "batch < 0");
    pa_status st = check_cache_shape(num_blocks, block_size, num_kv_heads, head_dim);
    if (st != PA_OK) return st;
    if ((st = check_heads(num_q_heads, num_kv_heads)) != PA_OK) return st;
    if (!(softmax_scale > 0.f) || !isfinite(softmax_scale))
        return fail(PA_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");
    if (batch == 0) return ok();
    if (max_context_len < 1) return fail(PA_ERR_INVALID_ARG, "max_context_len must be >= 1");
    if (block_table_stride < 1) return fail(PA_ERR_INVALID_ARG, "block_table_stride must be >= 1");
    if (num_splits < 0) return fail(PA_ERR_INVALID_ARG, "num_splits < 0");
    if (!out || !q || !k_cache || !v_cache || !block_table || !context_lens)
        return fail(PA_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(block_table, 4) || !aligned(context_lens, 4) || (dev_error && !aligned(dev_error, 4)))
        return fail(PA_ERR_INVALID_ARG, "misaligned pointer");
    if (fs) {
        const int64_t row = (int64_t)num_kv_heads * head_dim;
        if (!fs->k || !fs->v || !fs->slot_mapping) return fail(PA_ERR_INVALID_ARG, "NULL pointer");
        if (fs->k_row_stride < row || fs->v_row_stride < row)
            return fail(PA_ERR_INVALID_ARG, "row strides must be >= num_kv_heads * head_dim");
        if (fs->k_row_stride % 8 != 0 || fs->v_row_stride % 8 != 0 || !aligned(fs->k, 16) || !aligned(fs->v, 16))
            return fail(PA_ERR_UNSUPPORTED,
                        "the fused store needs 16-byte aligned k/v rows (row strides a multiple of 8 elements); "
                        "use pa_store_kv then pa_decode");
        if (!aligned(fs->slot_mapping, 4)) return fail(PA_ERR_INVALID_ARG, "misaligned pointer");
    }

    pa::DecodeArgs a = {};
    a.plan = pa::plan_decode(batch, num_kv_heads, max_context_len, num_splits, num_sms_current());
    if (a.plan.max_splits > pa::kDecodeMaxSplits || num_kv_heads > pa::kDecodeMaxKvHeads ||
        (int64_t)batch * num_kv_heads > pa::kDecodeMaxPairs)
        return fail(PA_ERR_UNSUPPORTED, "more than %d context splits, %d KV heads or %d (sequence, KV head) pairs",
                    pa::kDecodeMaxSplits, pa::kDecodeMaxKvHeads, pa::kDecodeMaxPairs);
    const pa::DecodeWorkspace wl = pa::decode_workspace_layout(a.plan, batch, num_q_heads, num_kv_heads, head_dim);
    const size_t need = wl.total;
    if (!workspace || workspace_bytes < need)
        return fail(PA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                    workspace ? workspace_bytes : (size_t)0);
    if (!aligned(workspace, 256)) return fail(PA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    a.out = out;
    a.q = q;
    a.block_table = block_table;
    a.context_lens = context_lens;
    a.dev_error = dev_error;
    char *ws = static_cast<char *>(workspace);
    a.plan_ws = ws + wl.plan_off;
    a.part_o = reinterpret_cast<float *>(ws + wl.o_off);
    a.part_lse = reinterpret_cast<float *>(ws + wl.lse_off);
    a.bt_stride = block_table_stride;
    a.batch = batch;
    a.num_q_heads = num_q_heads;
    a.num_kv_heads = num_kv_heads;
    a.group = num_q_heads / num_kv_heads;
    a.head_dim = head_dim;
    a.num_blocks = num_blocks;
    a.block_size = block_size;
    a.box_tokens = block_size < pa::kDecodeTileTokens ? block_size : pa::kDecodeTileTokens;
    a.max_context_len = max_context_len;
    a.scale_log2 = softmax_scale * 1.4426950408889634f;
    a.part_slots = a.plan.max_splits;
    a.part_base = 0;
    a.t_offset = 0;
    a.shared_blocks = 0;
    a.k_new = fs ? fs->k : nullptr;
    a.v_new = fs ? fs->v : nullptr;
    a.kn_stride = fs ? fs->k_row_stride : 0;
    a.vn_stride = fs ? fs->v_row_stride : 0;
    a.new_slots = fs ? fs->slot_mapping : nullptr;
    a.k_cache = const_cast<void *>(k_cache);
    a.v_cache = const_cast<void *>(v_cache);
    a.num_slots = (int64_t)num_blocks * block_size;

    CUtensorMap tm_k, tm_v;
    const int64_t rows = (int64_t)num_blocks * block_size;
    if ((st = encode_rows(&tm_k, k_cache, rows, num_kv_heads, head_dim, 1, a.box_tokens)) != PA_OK) return st;
    if ((st = encode_rows(&tm_v, v_cache, rows, num_kv_heads, head_dim, 1, a.box_tokens)) != PA_OK) return st;
    cudaError_t e = pa::launch_decode(a, tm_k, tm_v, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "decode kernel launch");
    return ok();
}

pa_status pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache, const int32_t *block_table,
                    int32_t block_table_stride, const int32_t *context_lens, int32_t batch, int32_t max_context_len,
                    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks,
                    int32_t block_size, float softmax_scale, void *workspace, size_t workspace_bytes,
                    int32_t *dev_error, void *stream) {
    return decode_impl(out, q, k_cache, v_cache, block_table, block_table_stride, context_lens, batch,
                       max_context_len, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size, softmax_scale,
                       0, workspace, workspace_bytes, dev_error, stream);
}

pa_status pa_store_kv_decode(const void *k, const void *v, int64_t k_row_stride, int64_t v_row_stride,
                             const int32_t *slot_mapping, void *out, const void *q, void *k_cache, void *v_cache,
                             const int32_t *block_table, int32_t block_table_stride, const int32_t *context_lens,
                             int32_t batch, int32_t max_context_len, int32_t num_q_heads, int32_t num_kv_heads,
                             int32_t head_dim, int32_t num_blocks, int32_t block_size, float softmax_scale,
                             void *workspace, size_t workspace_bytes, int32_t *dev_error, void *stream) {
    const FusedStore fs = {k, v, k_row_stride, v_row_stride, slot_mapping};
    return decode_impl(out, q, k_cache, v_cache, block_table, block_table_stride, context_lens, batch,
                       max_context_len, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size, softmax_scale,
                       0, workspace, workspace_bytes, dev_error, stream, &fs);
}

size_t pa_decode_split_workspace_size(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                      int32_t max_context_len, int32_t num_splits) {
    if (batch <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || max_context_len <= 0 ||
        num_splits < 0)
        return 0;
    pa::DecodePlan plan = pa::plan_decode(batch, num_kv_heads, max_context_len, num_splits, num_sms_current());
    return pa::decode_workspace_layout(plan, batch, num_q_heads, num_kv_heads, head_dim).total;
}

pa_status pa_decode_split(void *out, const void *q, const void *k_cache, const void *v_cache,
                          const int32_t *block_table, int32_t block_table_stride, const int32_t *context_lens,
                          int32_t batch, int32_t max_context_len, int32_t num_q_heads, int32_t num_kv_heads,
                          int32_t head_dim, int32_t num_blocks, int32_t block_size, float softmax_scale,
                          int32_t num_splits, void *workspace, size_t workspace_bytes, int32_t *dev_error,
                          void *stream) {
    return decode_impl(out, q, k_cache, v_cache, block_table, block_table_stride, context_lens, batch,
                       max_context_len, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size, softmax_scale,
                       num_splits, workspace, workspace_bytes, dev_error, stream);
}

}  // extern "C"

namespace {

// Work split of the shared-prefix decode: the prefix keys are cut into chunks so that the prefix phase
// has at most one work unit per SM; the private suffixes use the ordinary decode split.
struct SharedPlan {
    pa::DecodePlan dplan;
    int32_t nchunks, key_chunk, ranks, slots;
    size_t plan_bytes, o_bytes, lse_bytes, dplan_bytes, total;
};

SharedPlan plan_shared(int32_t batch, int32_t Hq, int32_t Hkv, int32_t D, int32_t max_ctx, int32_t B, int32_t P,
                       int sms) {
    SharedPlan sp;
    const int32_t G = Hq / Hkv, TQ = 128 / G;
    const int64_t nprefix = (int64_t)P * B;
    sp.ranks = (batch + 2 * TQ - 1) / (2 * TQ);
    const int64_t per_chunk_units = (int64_t)sp.ranks * Hkv;
    // at most one unit per SM: a unit of a few key tiles is mostly start-up, so a second round of units
    // costs more than the longer chunks of a single round
    int64_t nch = (int64_t)sms / per_chunk_units;
    const int64_t max_ch = (nprefix + 127) / 128;
    if (nch < 1) nch = 1;
    if (nch > max_ch) nch = max_ch;
    int64_t kc = (nprefix + nch - 1) / nch;
    kc = (kc + 127) / 128 * 128;
    sp.key_chunk = (int32_t)kc;
    sp.nchunks = (int32_t)((nprefix + kc - 1) / kc);
    const int32_t suffix = max_ctx - (int32_t)nprefix > 0 ? max_ctx - (int32_t)nprefix : 1;
    sp.dplan = pa::plan_decode(batch, Hkv, suffix, 0, sms);
    sp.slots = sp.nchunks + sp.dplan.max_splits;
    auto r256 = [](size_t x) { return (x + 255) / 256 * 256; };
    sp.plan_bytes = r256(pa::prefill_workspace_bytes(1, batch, G, Hkv, sp.nchunks));
    sp.o_bytes = r256((size_t)batch * Hq * sp.slots * D * sizeof(float));
    sp.lse_bytes = r256((size_t)batch * Hq * sp.slots * sizeof(float));
    // the suffix decode's item table (its partials are the slots after the prefix chunks, above)
    sp.dplan_bytes = pa::decode_plan_bytes(sp.dplan, batch, Hkv);
    sp.total = sp.plan_bytes + sp.o_bytes + sp.lse_bytes + sp.dplan_bytes;
    return sp;
}

}  // namespace

extern "C" {

size_t pa_decode_shared_prefix_workspace_size(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                              int32_t head_dim, int32_t max_context_len, int32_t block_size,
                                              int32_t num_shared_blocks) {
    if (batch <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 || head_dim <= 0 ||
        max_context_len <= 0 || block_size <= 0 || num_shared_blocks <= 0 ||
        128 % (num_q_heads / num_kv_heads) != 0)
        return 0;
    return plan_shared(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, block_size, num_shared_blocks,
                       num_sms_current())
        .total;
}

pa_status pa_decode_shared_prefix(void *out, const void *q, const void *k_cache, const void *v_cache,
                                  const int32_t *block_table, int32_t block_table_stride,
                                  const int32_t *context_lens, int32_t batch, int32_t max_context_len,
                                  int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks,
                                  int32_t block_size, float softmax_scale, int32_t num_shared_blocks,
                                  void *workspace, size_t workspace_bytes, int32_t *dev_error, void *stream) {
    if (batch < 0) return fail(PA_ERR_INVALID_ARG, "batch < 0");
    pa_status st = check_cache_shape(num_blocks, block_size, num_kv_heads, head_dim);
    if (st != PA_OK) return st;
    if ((st = check_heads(num_q_heads, num_kv_heads)) != PA_OK) return st;
    const int32_t G = num_q_heads / num_kv_heads;
    if (128 % G != 0) return fail(PA_ERR_UNSUPPORTED, "shared-prefix decode needs a GQA group that divides 128");
    if (!(softmax_scale > 0.f) || !isfinite(softmax_scale))
        return fail(PA_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");
    if (batch == 0) return ok();
    if (max_context_len < 1 || block_table_stride < 1) return fail(PA_ERR_INVALID_ARG, "bad max_context_len or stride");
    if (num_shared_blocks < 1 || num_shared_blocks > block_table_stride ||
        (int64_t)num_shared_blocks * block_size > max_context_len)
        return fail(PA_ERR_INVALID_ARG, "num_shared_blocks must be in [1, stride] and cover at most max_context_len");
    if (batch > 65535 * 64) return fail(PA_ERR_UNSUPPORTED, "batch too large");
    if (!out || !q || !k_cache || !v_cache || !block_table || !context_lens)
        return fail(PA_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(block_table, 4) || !aligned(context_lens, 4) || (dev_error && !aligned(dev_error, 4)))
        return fail(PA_ERR_INVALID_ARG, "misaligned pointer");
    const int sms = num_sms_current();
    const SharedPlan sp = plan_shared(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, block_size,
                                      num_shared_blocks, sms);
    if (!workspace || workspace_bytes < sp.total)
        return fail(PA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", sp.total,
                    workspace ? workspace_bytes : (size_t)0);
    if (!aligned(workspace, 256)) return fail(PA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    char *ws = static_cast<char *>(workspace);
    float *part_o = reinterpret_cast<float *>(ws + sp.plan_bytes);
    float *part_lse = reinterpret_cast<float *>(ws + sp.plan_bytes + sp.o_bytes);
    const int64_t rows = (int64_t)num_blocks * block_size;
    const int32_t nprefix = num_shared_blocks * block_size;
    cudaStream_t str = static_cast<cudaStream_t>(stream);

    // 1. prefix: every query of the batch against the shared blocks (row 0 of the table), non-causal,
    //    as one prefill "sequence" of `batch` query rows; fp32 partials per key chunk
    pa::PrefillArgs pf = {};
    pf.q = q;
    pf.cu_q = pf.cu_k = nullptr;
    pf.block_table = block_table;
    pf.dev_error = dev_error;
    pf.bt_stride = block_table_stride;
    pf.batch = 1;
    pf.num_q_heads = num_q_heads;
    pf.num_kv_heads = num_kv_heads;
    pf.group = G;
    pf.head_dim = head_dim;
    pf.num_blocks = num_blocks;
    pf.block_size = block_size;
    pf.box_tokens = block_size < 128 ? block_size : 128;
    pf.max_seqlen_q = batch;
    pf.max_seqlen_k = nprefix;
    pf.causal = 0;
    pf.total_q = batch;
    pf.ranks = sp.ranks;
    pf.workspace = ws;
    pf.scale_log2 = softmax_scale * 1.4426950408889634f;
    pf.single_n_new = batch;
    pf.single_n_k = nprefix;
    pf.key_chunk = sp.key_chunk;
    pf.nchunks = sp.nchunks;
    pf.part_o = part_o;
    pf.part_lse = part_lse;
    pf.part_slots = sp.slots;
    pf.part_base = 0;
    CUtensorMap tq, tk, tv;
    if ((st = encode_rows(&tq, q, batch, num_q_heads, head_dim, G, 128 / G)) != PA_OK) return st;
    if ((st = encode_rows(&tk, k_cache, rows, num_kv_heads, head_dim, 1, pf.box_tokens)) != PA_OK) return st;
    if ((st = encode_rows(&tv, v_cache, rows, num_kv_heads, head_dim, 1, pf.box_tokens)) != PA_OK) return st;
    cudaError_t e = pa::launch_prefill(pf, tq, tk, tv, str);
    if (e != cudaSuccess) return cuda_fail(e, "shared-prefix kernel launch");

    // 2. private suffixes: split-KV decode from token nprefix on, partials after the prefix chunks;
    // 3. the combine kernel merges all partials of each (sequence, q-head)
    if (sp.dplan.max_splits > pa::kDecodeMaxSplits || num_kv_heads > pa::kDecodeMaxKvHeads ||
        (int64_t)batch * num_kv_heads > pa::kDecodeMaxPairs)
        return fail(PA_ERR_UNSUPPORTED, "more than %d context splits, %d KV heads or %d (sequence, KV head) pairs",
                    pa::kDecodeMaxSplits, pa::kDecodeMaxKvHeads, pa::kDecodeMaxPairs);
    pa::DecodeArgs da = {};
    da.plan = sp.dplan;
    da.out = out;
    da.q = q;
    da.block_table = block_table;
    da.context_lens = context_lens;
    da.dev_error = dev_error;
    da.part_o = part_o;
    da.part_lse = part_lse;
    da.plan_ws = ws + sp.plan_bytes + sp.o_bytes + sp.lse_bytes;
    da.bt_stride = block_table_stride;
    da.batch = batch;
    da.num_q_heads = num_q_heads;
    da.num_kv_heads = num_kv_heads;
    da.group = G;
    da.head_dim = head_dim;
    da.num_blocks = num_blocks;
    da.block_size = block_size;
    da.box_tokens = block_size < pa::kDecodeTileTokens ? block_size : pa::kDecodeTileTokens;
    da.max_context_len = max_context_len;
    da.scale_log2 = pf.scale_log2;
    da.part_slots = sp.slots;
    da.part_base = sp.nchunks;
    da.t_offset = nprefix;
    da.shared_blocks = num_shared_blocks;
    da.num_slots = rows;
    CUtensorMap dk, dv;
    if ((st = encode_rows(&dk, k_cache, rows, num_kv_heads, head_dim, 1, da.box_tokens)) != PA_OK) return st;
    if ((st = encode_rows(&dv, v_cache, rows, num_kv_heads, head_dim, 1, da.box_tokens)) != PA_OK) return st;
    e = pa::launch_decode(da, dk, dv, str);
    if (e != cudaSuccess) return cuda_fail(e, "shared-prefix suffix decode launch");
    return ok();
}

size_t pa_prefill_workspace_size(int32_t batch, int32_t max_seqlen_q, int32_t num_q_heads, int32_t num_kv_heads,
                                 int32_t head_dim) {
    (void)head_dim;
    if (batch <= 0 || max_seqlen_q <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 ||
        num_q_heads % num_kv_heads != 0 || 128 % (num_q_heads / num_kv_heads) != 0)
        return 0;
    return pa::prefill_workspace_bytes(batch, max_seqlen_q, num_q_heads / num_kv_heads, num_kv_heads);
}

static pa_status prefill_impl(void *out, const void *q, int32_t total_q, const void *k_cache, const void *v_cache,
                              const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, int32_t max_seqlen_q,
                              int32_t max_seqlen_k, const int32_t *block_table, int32_t block_table_stride,
                              int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                              int32_t num_blocks, int32_t block_size, float softmax_scale, int32_t causal,
                              void *workspace, size_t workspace_bytes, int32_t *dev_error, void *stream,
                              const FusedStore *fs, int32_t skip_single = 0) {
    if (batch < 0) return fail(PA_ERR_INVALID_ARG, "batch < 0");
    pa_status st = check_cache_shape(num_blocks, block_size, num_kv_heads, head_dim);
    if (st != PA_OK) return st;
    if ((st = check_heads(num_q_heads, num_kv_heads)) != PA_OK) return st;
    if (128 % (num_q_heads / num_kv_heads) != 0)
        return fail(PA_ERR_UNSUPPORTED, "prefill needs a GQA group that divides 128");
    if (!(softmax_scale > 0.f) || !isfinite(softmax_scale))
        return fail(PA_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");
    if (total_q < 0) return fail(PA_ERR_INVALID_ARG, "total_q < 0");
    if (batch == 0 || max_seqlen_q == 0 || total_q == 0) return ok();
    if (max_seqlen_q < 0 || max_seqlen_k < 1 || max_seqlen_k < max_seqlen_q)
        return fail(PA_ERR_INVALID_ARG, "need 0 <= max_seqlen_q <= max_seqlen_k and max_seqlen_k >= 1");
    if (block_table_stride < 1) return fail(PA_ERR_INVALID_ARG, "block_table_stride must be >= 1");
    if (batch > pa::kPrefillMaxBatch) return fail(PA_ERR_UNSUPPORTED, "batch > %d", pa::kPrefillMaxBatch);
    {
        const size_t need = pa::prefill_workspace_bytes(batch, max_seqlen_q, num_q_heads / num_kv_heads, num_kv_heads);
        if (!workspace || workspace_bytes < need)
            return fail(PA_ERR_WORKSPACE, "prefill workspace of %zu bytes needed, %zu given", need,
                        workspace ? workspace_bytes : (size_t)0);
        if (!aligned(workspace, 256)) return fail(PA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    }
    if (!out || !q || !k_cache || !v_cache || !cu_seqlens_q || !cu_seqlens_k || !block_table)
        return fail(PA_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(cu_seqlens_q, 4) || !aligned(cu_seqlens_k, 4) || !aligned(block_table, 4) ||
        (dev_error && !aligned(dev_error, 4)))
        return fail(PA_ERR_INVALID_ARG, "misaligned pointer");
    if (fs) {
        const int64_t row = (int64_t)num_kv_heads * head_dim;
        if (!fs->k || !fs->v || !fs->slot_mapping) return fail(PA_ERR_INVALID_ARG, "NULL pointer");
        if (fs->k_row_stride < row || fs->v_row_stride < row)
            return fail(PA_ERR_INVALID_ARG, "row strides must be >= num_kv_heads * head_dim");
        if (fs->k_row_stride % 8 != 0 || fs->v_row_stride % 8 != 0 || !aligned(fs->k, 16) || !aligned(fs->v, 16))
            return fail(PA_ERR_UNSUPPORTED,
                        "the fused store needs 16-byte aligned k/v rows (row strides a multiple of 8 elements); "
                        "use pa_store_kv then pa_prefill_varlen");
        if (!aligned(fs->slot_mapping, 4)) return fail(PA_ERR_INVALID_ARG, "misaligned pointer");
    }

    pa::PrefillArgs a = {};
    a.out = out;
    a.q = q;
    a.cu_q = cu_seqlens_q;
    a.cu_k = cu_seqlens_k;
    a.block_table = block_table;
    a.dev_error = dev_error;
    a.bt_stride = block_table_stride;
    a.batch = batch;
    a.num_q_heads = num_q_heads;
    a.num_kv_heads = num_kv_heads;
    a.group = num_q_heads / num_kv_heads;
    a.head_dim = head_dim;
    a.num_blocks = num_blocks;
    a.block_size = block_size;
    a.box_tokens = block_size < 128 ? block_size : 128;
    a.max_seqlen_q = max_seqlen_q;
    a.max_seqlen_k = max_seqlen_k;
    a.causal = causal ? 1 : 0;
    a.total_q = total_q;
    a.ranks = (max_seqlen_q + 2 * (128 / a.group) - 1) / (2 * (128 / a.group));
    a.workspace = workspace;
    a.single_n_new = a.single_n_k = 0;
    a.key_chunk = 0;
    a.nchunks = 1;
    a.part_o = a.part_lse = nullptr;
    a.part_slots = a.part_base = 0;
    a.skip_single = skip_single;
    a.scale_log2 = softmax_scale * 1.4426950408889634f;

    CUtensorMap tm_k, tm_v;
    const int64_t rows = (int64_t)num_blocks * block_size;
    if ((st = encode_rows(&tm_k, k_cache, rows, num_kv_heads, head_dim, 1, a.box_tokens)) != PA_OK) return st;
    if ((st = encode_rows(&tm_v, v_cache, rows, num_kv_heads, head_dim, 1, a.box_tokens)) != PA_OK) return st;
    // q viewed as [total_q, Hq, D]: one box is the (128 / G) tokens x G q-heads of one Q tile
    CUtensorMap tm_q;
    if ((st = encode_rows(&tm_q, q, total_q, num_q_heads, head_dim, a.group, 128 / a.group)) != PA_OK) return st;
    CUtensorMap tm_kn, tm_vn;
    if (fs) {
        a.k_new = fs->k;
        a.v_new = fs->v;
        a.kn_stride = fs->k_row_stride;
        a.vn_stride = fs->v_row_stride;
        a.new_slots = fs->slot_mapping;
        a.k_cache = const_cast<void *>(k_cache);
        a.v_cache = const_cast<void *>(v_cache);
        a.num_slots = rows;
        // the new K/V rows as [total_q, Hkv, D] with their row strides, boxes as the cache's
        if ((st = encode_rows(&tm_kn, fs->k, total_q, num_kv_heads, head_dim, 1, a.box_tokens, fs->k_row_stride)) !=
            PA_OK)
            return st;
        if ((st = encode_rows(&tm_vn, fs->v, total_q, num_kv_heads, head_dim, 1, a.box_tokens, fs->v_row_stride)) !=
            PA_OK)
            return st;
    }
    cudaError_t e = pa::launch_prefill(a, tm_q, tm_k, tm_v, static_cast<cudaStream_t>(stream), fs ? &tm_kn : nullptr,
                                       fs ? &tm_vn : nullptr);
    if (e == cudaErrorNotSupported) return fail(PA_ERR_UNSUPPORTED, "prefill kernel not available");
    if (e != cudaSuccess) return cuda_fail(e, "prefill kernel launch");
    return ok();
}

pa_status pa_prefill_varlen(void *out, const void *q, int32_t total_q, const void *k_cache, const void *v_cache,
                            const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, int32_t max_seqlen_q,
                            int32_t max_seqlen_k, const int32_t *block_table, int32_t block_table_stride,
                            int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                            int32_t num_blocks, int32_t block_size, float softmax_scale, int32_t causal,
                            void *workspace, size_t workspace_bytes, int32_t *dev_error, void *stream) {
    return prefill_impl(out, q, total_q, k_cache, v_cache, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                        block_table, block_table_stride, batch, num_q_heads, num_kv_heads, head_dim, num_blocks,
                        block_size, softmax_scale, causal, workspace, workspace_bytes, dev_error, stream, nullptr);
}

size_t pa_prefill_varlen_mixed_workspace_size(int32_t batch, int32_t max_seqlen_q, int32_t max_seqlen_k,
                                              int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim) {
    if (batch <= 0 || max_seqlen_q <= 0 || max_seqlen_k <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 ||
        num_q_heads % num_kv_heads != 0 || 128 % (num_q_heads / num_kv_heads) != 0 || head_dim <= 0)
        return 0;
    const size_t pf = (pa::prefill_workspace_bytes(batch, max_seqlen_q, num_q_heads / num_kv_heads, num_kv_heads) +
                       255) / 256 * 256;
    const pa::DecodePlan plan = pa::plan_decode(batch, num_kv_heads, max_seqlen_k, 0, num_sms_current());
    return pf + pa::decode_workspace_layout(plan, batch, num_q_heads, num_kv_heads, head_dim).total;
}

pa_status pa_prefill_varlen_mixed(void *out, const void *q, int32_t total_q, const void *k_cache, const void *v_cache,
                                  const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, int32_t max_seqlen_q,
                                  int32_t max_seqlen_k, const int32_t *block_table, int32_t block_table_stride,
                                  int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                  int32_t num_blocks, int32_t block_size, float softmax_scale, void *workspace,
                                  size_t workspace_bytes, int32_t *dev_error, void *stream) {
    if (batch < 0) return fail(PA_ERR_INVALID_ARG, "batch < 0");
    if (batch == 0 || max_seqlen_q == 0 || total_q == 0)   // (the prefill call below validates the rest)
        return prefill_impl(out, q, total_q, k_cache, v_cache, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                            max_seqlen_k, block_table, block_table_stride, batch, num_q_heads, num_kv_heads, head_dim,
                            num_blocks, block_size, softmax_scale, 1, workspace, workspace_bytes, dev_error, stream,
                            nullptr, 1);
    pa_status st = check_heads(num_q_heads, num_kv_heads);
    if (st != PA_OK) return st;
    if (max_seqlen_k < 1 || max_seqlen_q < 0 || head_dim < 1)
        return fail(PA_ERR_INVALID_ARG, "need max_seqlen_k >= 1 and head_dim >= 1");
    const size_t need = pa_prefill_varlen_mixed_workspace_size(batch, max_seqlen_q, max_seqlen_k, num_q_heads,
                                                               num_kv_heads, head_dim);
    if (need == 0) return fail(PA_ERR_UNSUPPORTED, "shape not supported (the GQA group must divide 128)");
    if (!workspace || workspace_bytes < need)
        return fail(PA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                    workspace ? workspace_bytes : (size_t)0);
    if (!aligned(workspace, 256)) return fail(PA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    const size_t pf_bytes =
        (pa::prefill_workspace_bytes(batch, max_seqlen_q, num_q_heads / num_kv_heads, num_kv_heads) + 255) / 256 * 256;
    // 1. the prompts (every sequence with more than one new token): the prefill kernel; it validates
    //    every argument before anything is enqueued
    st = prefill_impl(out, q, total_q, k_cache, v_cache, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                      block_table, block_table_stride, batch, num_q_heads, num_kv_heads, head_dim, num_blocks,
                      block_size, softmax_scale, 1, workspace, pf_bytes, dev_error, stream, nullptr, 1);
    if (st != PA_OK) return st;
    // 2. the decode rows (one new token, context n_k): the split-KV decode in its varlen mode
    pa::DecodeArgs da = {};
    da.plan = pa::plan_decode(batch, num_kv_heads, max_seqlen_k, 0, num_sms_current());
    if (da.plan.max_splits > pa::kDecodeMaxSplits || num_kv_heads > pa::kDecodeMaxKvHeads ||
        (int64_t)batch * num_kv_heads > pa::kDecodeMaxPairs)
        return fail(PA_ERR_UNSUPPORTED, "more than %d context splits, %d KV heads or %d (sequence, KV head) pairs",
                    pa::kDecodeMaxSplits, pa::kDecodeMaxKvHeads, pa::kDecodeMaxPairs);
    const pa::DecodeWorkspace wl = pa::decode_workspace_layout(da.plan, batch, num_q_heads, num_kv_heads, head_dim);
    char *ws = static_cast<char *>(workspace) + pf_bytes;
    da.plan_ws = ws + wl.plan_off;
    da.part_o = reinterpret_cast<float *>(ws + wl.o_off);
    da.part_lse = reinterpret_cast<float *>(ws + wl.lse_off);
    da.out = out;
    da.q = q;
    da.block_table = block_table;
    da.context_lens = nullptr;
    da.vl_cu_q = cu_seqlens_q;
    da.vl_cu_k = cu_seqlens_k;
    da.dev_error = dev_error;
    da.bt_stride = block_table_stride;
    da.batch = batch;
    da.num_q_heads = num_q_heads;
    da.num_kv_heads = num_kv_heads;
    da.group = num_q_heads / num_kv_heads;
    da.head_dim = head_dim;
    da.num_blocks = num_blocks;
    da.block_size = block_size;
    da.box_tokens = block_size < pa::kDecodeTileTokens ? block_size : pa::kDecodeTileTokens;
    da.max_context_len = max_seqlen_k;
    da.scale_log2 = softmax_scale * 1.4426950408889634f;
    da.part_slots = da.plan.max_splits;
    da.part_base = 0;
    da.t_offset = 0;
    da.num_slots = (int64_t)num_blocks * block_size;
    CUtensorMap dk, dv;
    const int64_t rows = (int64_t)num_blocks * block_size;
    if ((st = encode_rows(&dk, k_cache, rows, num_kv_heads, head_dim, 1, da.box_tokens)) != PA_OK) return st;
    if ((st = encode_rows(&dv, v_cache, rows, num_kv_heads, head_dim, 1, da.box_tokens)) != PA_OK) return st;
    cudaError_t e = pa::launch_decode(da, dk, dv, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "mixed-batch decode launch");
    return ok();
}

pa_status pa_store_kv_prefill_varlen(const void *k, const void *v, int64_t k_row_stride, int64_t v_row_stride,
                                     const int32_t *slot_mapping, void *out, const void *q, int32_t total_q,
                                     void *k_cache, void *v_cache, const int32_t *cu_seqlens_q,
                                     const int32_t *cu_seqlens_k, int32_t max_seqlen_q, int32_t max_seqlen_k,
                                     const int32_t *block_table, int32_t block_table_stride, int32_t batch,
                                     int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks,
                                     int32_t block_size, float softmax_scale, int32_t causal, void *workspace,
                                     size_t workspace_bytes, int32_t *dev_error, void *stream) {
    const FusedStore fs = {k, v, k_row_stride, v_row_stride, slot_mapping};
    return prefill_impl(out, q, total_q, k_cache, v_cache, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                        block_table, block_table_stride, batch, num_q_heads, num_kv_heads, head_dim, num_blocks,
                        block_size, softmax_scale, causal, workspace, workspace_bytes, dev_error, stream, &fs);
}

pa_status pa_selftest_bounded_wait(int32_t *dev_error, int64_t max_polls, void *stream) {
    if (!dev_error || !aligned(dev_error, 4)) return fail(PA_ERR_INVALID_ARG, "dev_error must be a device int32");
    if (max_polls < 1 || max_polls > (int64_t(1) << 30)) return fail(PA_ERR_INVALID_ARG, "max_polls out of range");
    cudaError_t e = pa::launch_selftest_wait(dev_error, max_polls, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
    return ok();
}

pa_status pa_selftest_exp2(const float *x, float *y_poly, float *y_sfu, int32_t n, void *stream) {
    if (n < 0) return fail(PA_ERR_INVALID_ARG, "n < 0");
    if (n == 0) return ok();
    if (!x || !y_poly || !y_sfu || !aligned(x, 4) || !aligned(y_poly, 4) || !aligned(y_sfu, 4))
        return fail(PA_ERR_INVALID_ARG, "x, y_poly and y_sfu must be float arrays in device memory");
    cudaError_t e = pa::launch_selftest_exp2(x, y_poly, y_sfu, n, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
    return ok();
}

}  // extern "C"
