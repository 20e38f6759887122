// Paged GQA decode attention: split-KV flash-decoding plus a combine pass,
// optionally with this step's store_kvcache fused into the split kernel.
//
// What it computes (per sequence s, q-head h):
//     out[s, h] = softmax_j(scale * q[s, h] . K_j) V_j  over the context of s,
// the attention formula of the chenxutan.com Nano-vLLM article (section 1.2),
// K_j / V_j taken from KV head h / G (GQA, same article, section 3.2.1) and
// gathered through block_table (gsyq.cn article, sections 4.1 and 5.3) -- the
// flash_attn_with_kvcache call of the nano-vllm walkthrough (section seven).
//
// How:
//  * a one-CTA planning kernel writes a longest-first table of work items; an
//    item is a token range of one sequence's context (all of it, or one split
//    of a context far longer than the average per-CTA load) for one KV head
//    and ALL G q-heads of its GQA group, so every K/V byte is read from HBM
//    once per call.  Persistent CTAs (2 per SM) take items with an atomic
//    counter and stream them through one continuous TMA ring.
//  * warp 4 is a TMA producer: it fetches the next item, hands it to the
//    consumers with the item's Q rows, and for each 64-token tile it reads the tile's
//    physical block ids from block_table and issues 3-D tensor-map loads
//    (128-byte swizzle) of the K and V rows of this KV head into a 3-stage
//    shared-memory ring guarded by mbarriers.
//  * warps 0-3 each take 16 tokens of a tile: S = Q K^T and O += P V on the
//    tensor cores with mma.sync m16n8k16 (bf16 in, fp32 accumulate), the G
//    q-heads padded to the 16 rows of the A operand, online softmax in fp32
//    (base-2 exponent, scale * log2(e) folded into the scores).
//  * the four warps' (max, sum, O) are merged in shared memory; with one split
//    the CTA writes bf16 out, otherwise a normalised fp32 partial and its
//    log-sum-exp go to the workspace and decode_combine_kernel merges them.
//  * masked positions (past the end of the context) are selected out: their
//    score becomes -inf and their V rows are zeroed in registers, so stale or
//    poisoned cache contents never reach the result (0 * NaN is never formed).
//  * fused store (pa_store_kv_decode): the consumer warp whose 16-token slice
//    holds position context_len - 1 of the pair's last split copies the new
//    token's K/V row of its KV head into a staging row at the start of the
//    item (cp.async), and, once the tile holding that position has landed,
//    writes it into the tile in shared memory (in place of the cache row the
//    TMA brought) and to its cache slot in HBM -- the store_kvcache of the
//    walkthrough, section seven, done inside the attention launch.
//  * varlen mode (pa_prefill_varlen_mixed): the decode rows of a batch that
//    mixes decode steps with prompts -- sequence s is this call's work only if
//    it has one new token; its q / out row is cu_seqlens_q[s] and its context
//    n_k.
#include <float.h>

#include <atomic>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr int kTile = kDecodeTileTokens;  // tokens per pipeline stage
constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kHalfBytes = kTile * 128;   // one 64-element slice of head_dim for 64 tokens

template <int D>
struct DecodeCfg {
    static constexpr int kHalves = D / 64;
    static constexpr int kStages = D == 128 ? 3 : 6;
    static constexpr int kKvBytes = kHalves * kHalfBytes;        // K (or V) part of a stage
    static constexpr int kStageBytes = 2 * kKvBytes;
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kBarOff = kRingBytes;                   // 256 bytes of barriers
    static constexpr int kNewOff = kBarOff + 256;                // fused store: the new token's K and V row
    static constexpr int kQOff = kNewOff + 512;                  // 2 slots of the group's G q-head rows
    // then the merge area: per consumer warp, G rows of D partial sums plus (max, sum)
    static constexpr size_t red_off(int G) { return (size_t)kQOff + 2 * (size_t)G * D * 2; }
    static constexpr size_t smem_bytes(int G) {
        return red_off(G) + (size_t)kConsumerWarps * G * (D + 2) * 4 + 1024;
    }
};

__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
}

// Work items.  The planning kernel (decode_plan_kernel, one CTA, run first) reads the context lengths and
// writes a table of items (sequence, KV head, split, token range) into the workspace, ordered from the
// longest to the shortest, plus a hand-out counter.  A pair (sequence, KV head) whose context is at most
// `whole` tiles is one item; a longer one is cut into splits of `chunk` tiles.  `whole` is the average
// per-CTA load, so on a mix of lengths (the Qwen3-like workload) nothing is split and no partial is written,
// and pairs far longer than the average (long context) are cut fine enough to balance.  Persistent CTAs
// take items from the table with an atomic counter: the longest first, so the short ones fill the tail.
struct DecPlanHdr {
    int32_t counter;       // next item to hand out
    int32_t n_items;
    int32_t whole;         // tiles: a pair of at most this many tiles is one item (0: always split)
    int32_t chunk;         // tiles per split of a longer pair
};
constexpr int kPlanHdrBytes = 256;
constexpr int kDecSkip = -2;                // item.x of a first slot whose pair has no work (CTA takes the counter's)
constexpr int kPlanThreads = 1024;
constexpr int kPlanBuckets = 1024;
constexpr int kDecLocalCut = 1024;          // batches up to this many sequences: each CTA cuts its first item itself          // item lengths (tiles) for the longest-first order; longer share the last
constexpr int kPlanCache = 2048;            // sequences whose length the planning kernel keeps in shared memory
constexpr int kPlanSplitList = 1024;        // split (sequence, KV head) pairs whose items a warp each writes

// Context length of sequence s: context_lens[s]; in the varlen mode (the decode rows of a mixed batch) the
// key count of a sequence with exactly one new token, and -1 for any other sequence (not this call's work).
__device__ __forceinline__ int dec_ctx(const DecodeArgs &a, int s) {
    if (!a.vl_cu_q) return __ldg(a.context_lens + s);
    if (__ldg(a.vl_cu_q + s + 1) - __ldg(a.vl_cu_q + s) != 1) return -1;
    return __ldg(a.vl_cu_k + s + 1) - __ldg(a.vl_cu_k + s);
}

// Row of sequence s in q and out.
__device__ __forceinline__ int64_t dec_row(const DecodeArgs &a, int s) {
    return a.vl_cu_q ? (int64_t)__ldg(a.vl_cu_q + s) : (int64_t)s;
}

// Item: {s, kvh | split << 16, t_begin, t_end}; s < 0 marks the end of the stream in shared memory.
__device__ __forceinline__ int dec_tiles(const DecodeArgs &a, int s, bool report_bad) {
    const int ctx = dec_ctx(a, s);
    if (ctx == -1) return 0;                  // a prefill sequence of a mixed batch
    if (ctx < 1 || ctx > a.max_context_len || (int64_t)ctx > (int64_t)a.bt_stride * a.block_size ||
        ctx < a.t_offset) {
        if (report_bad) report(a.dev_error, PA_DEVERR_CONTEXT_LEN);
        return 0;
    }
    return (ctx - a.t_offset + kTile - 1) / kTile;
}

// How a pair of `tiles` tiles is cut under (whole, chunk).  At most `whole` tiles: one item.  Longer: pieces of
// `chunk` tiles, except that the last two chunks' worth (the remainder included) is cut into kTailPieces
// smaller pieces, so that the items handed out last -- the shortest, in the longest-first order -- are small
// and the CTAs finish together.  whole == 0 (a split count the caller fixed): uniform pieces of `chunk`.
constexpr int kTailPieces = 4;
struct SplitGeom {
    int n;       // splits
    int nfull;   // leading splits of `chunk` tiles
    int np;      // tail pieces after them: `base` tiles, the first `extra` of them one more
    int base, extra;
};
__device__ __forceinline__ SplitGeom dec_split_geom(int tiles, int whole, int chunk) {
    SplitGeom g;
    g.n = g.nfull = g.np = g.base = g.extra = 0;
    if (tiles == 0) return g;
    if (tiles <= whole) {
        g.n = 1;
        g.np = 1;
        g.base = tiles;
        return g;
    }
    const int n = (tiles + chunk - 1) / chunk;
    g.nfull = whole == 0 || n < 2 ? n - 1 : n - 2;
    const int tail = tiles - g.nfull * chunk;
    g.np = whole == 0 || n < 2 ? 1 : min(kTailPieces, tail);
    g.base = tail / g.np;
    g.extra = tail - g.base * g.np;
    g.n = g.nfull + g.np;
    return g;
}
__device__ __forceinline__ int dec_nsplit(int tiles, int whole, int chunk) {
    return dec_split_geom(tiles, whole, chunk).n;
}
// First tile of split j (j == n: the end).
__device__ __forceinline__ int dec_split_begin(const SplitGeom &g, int chunk, int j) {
    if (j <= g.nfull) return j * chunk;
    const int k = j - g.nfull;
    return g.nfull * chunk + k * g.base + min(k, g.extra);
}

// The split rule, from the total work in tiles over the grid's CTAs: pairs up to the average per-CTA load stay
// whole; longer ones are cut into pieces of a quarter of it (never finer than the host's chunk, which sized the
// partial slots; an eighth measured 2 us slower at long context: more partials to merge, and the tail pieces
// already even out the ends).  The planning kernel and each decode CTA (for its first item) apply it to the
// same total, so they cut every pair the same way.
__device__ __forceinline__ void dec_cut(const DecodeArgs &a, unsigned long long total, int num_ctas, int &whole,
                                        int &chunk) {
    const int host_chunk = a.plan.chunk / kTile;
    if (a.plan.fixed) {
        whole = 0;
        chunk = host_chunk;
        return;
    }
    const unsigned long long avg = (total + num_ctas - 1) / (unsigned long long)num_ctas;
    whole = (int)min(avg, 1ull << 30);
    if (whole < 4) whole = 4;
    chunk = (int)min((avg + 3) / 4, 1ull << 30);
    if (chunk < host_chunk) chunk = host_chunk;
}

// Total work of the call in tiles: every (sequence, KV head) pair's tiles past t_offset.  Summed by the 32 lanes
// of a warp (the planning kernel sums the same values over its threads).
__device__ __forceinline__ unsigned long long dec_total_warp(const DecodeArgs &a, int lane) {
    unsigned long long part = 0;
    for (int s = lane; s < a.batch; s += 32) part += (unsigned long long)dec_tiles(a, s, false) * a.num_kv_heads;
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    return part;
}

// Output rows of (sequence s, KV head kvh) from its part_base partials alone (no tile of its own): the
// element loop is strided over `nthreads` threads starting at `t0`.
__device__ void plan_merge_bare(const DecodeArgs &a, int s, int kvh, int t0, int nthreads) {
    const int G = a.group, D = a.head_dim;
    for (int e = t0; e < G * D; e += nthreads) {
        const int g = e / D, d = e % D, h = kvh * G + g;
        const int64_t pb = ((int64_t)s * a.num_q_heads + h) * a.part_slots;
        float m = -INFINITY;
        for (int j = 0; j < a.part_base; ++j) m = fmaxf(m, __ldcg(a.part_lse + pb + j));
        float num = 0.f, den = 0.f;
        for (int j = 0; j < a.part_base; ++j) {
            const float w = fast_exp2(__ldcg(a.part_lse + pb + j) - m);
            num += w * __ldcg(a.part_o + (pb + j) * D + d);
            den += w;
        }
        static_cast<__nv_bfloat16 *>(a.out)[(dec_row(a, s) * a.num_q_heads + h) * D + d] = __float2bfloat16_rn(num / den);
    }
}

__global__ void __launch_bounds__(kPlanThreads) decode_plan_kernel(const DecodeArgs a, int32_t num_ctas) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");   // the decode kernel may start its set-up
    __shared__ unsigned long long s_total;
    __shared__ int s_off[kPlanBuckets];
    // tiles and context length of the first kPlanCache sequences, read once from global memory
    __shared__ int s_tiles[kPlanCache], s_ctx[kPlanCache];
    const int tid = threadIdx.x;
    if (tid == 0) s_total = 0;
    for (int b = tid; b < kPlanBuckets; b += kPlanThreads) s_off[b] = 0;
    __syncthreads();
    // total work in tiles; checked mode: context lengths and the shared blocks
    unsigned long long part = 0;
    for (int s = tid; s < a.batch; s += kPlanThreads) {
        const int tiles = dec_tiles(a, s, true);
        if (s < kPlanCache) {
            s_tiles[s] = tiles;
            s_ctx[s] = dec_ctx(a, s);
        }
        part += (unsigned long long)tiles * a.num_kv_heads;
        if (a.dev_error && a.shared_blocks > 0)
            for (int b = 0; b < a.shared_blocks; ++b)
                if (__ldg(a.block_table + (int64_t)s * a.bt_stride + b) != __ldg(a.block_table + b))
                    report(a.dev_error, PA_DEVERR_BLOCK_ID);
    }
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if ((tid & 31) == 0) atomicAdd(&s_total, part);
    __syncthreads();
    int whole, chunk;
    dec_cut(a, s_total, num_ctas, whole, chunk);
    // Item order: slots 0 .. n_first-1 hold the first split of pairs 0 .. n_first-1 (CTA c's first item, which
    // its producer starts loading before this table exists), then every other item longest first: count those
    // per length bucket, then exclusive offsets from the longest bucket
    const int n_first = min(num_ctas, a.batch * a.num_kv_heads);
    auto bucket = [](int tiles) { return min(tiles, kPlanBuckets - 1); };
    for (int s = tid; s < a.batch; s += kPlanThreads) {
        const int tiles = s < kPlanCache ? s_tiles[s] : dec_tiles(a, s, false);
        const SplitGeom g = dec_split_geom(tiles, whole, chunk);
        if (g.n == 0) continue;
        if (g.nfull > 0) atomicAdd(&s_off[bucket(chunk)], g.nfull * a.num_kv_heads);
        if (g.extra > 0) atomicAdd(&s_off[bucket(g.base + 1)], g.extra * a.num_kv_heads);
        atomicAdd(&s_off[bucket(g.base)], (g.np - g.extra) * a.num_kv_heads);
        const int nf = min(max(n_first - s * a.num_kv_heads, 0), a.num_kv_heads);   // first pairs of sequence s
        if (nf > 0) atomicAdd(&s_off[bucket(dec_split_begin(g, chunk, 1))], -nf);
    }
    __syncthreads();
    {   // exclusive scan over the buckets from the longest down: thread t owns bucket kPlanBuckets - 1 - t
        static_assert(kPlanBuckets == kPlanThreads, "one bucket per thread");
        __shared__ int s_warp[kPlanThreads / 32];
        const int b = kPlanBuckets - 1 - tid, lane = tid & 31, w = tid >> 5;
        const int v = s_off[b];
        int inc = v;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        if (lane == 31) s_warp[w] = inc;
        __syncthreads();
        if (w == 0) {
            int t = s_warp[lane];
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, t, o);
                if (lane >= o) t += y;
            }
            s_warp[lane] = t;               // inclusive totals of warps 0..lane
        }
        __syncthreads();
        s_off[b] = n_first + inc - v + (w > 0 ? s_warp[w - 1] : 0);
        if (tid == kPlanThreads - 1) {
            DecPlanHdr *h = reinterpret_cast<DecPlanHdr *>(a.plan_ws);
            h->counter = n_first;           // item c < n_first is CTA c's first item (taken without the counter)
            h->n_items = n_first + s_warp[kPlanThreads / 32 - 1];
            h->whole = whole;
            h->chunk = chunk;
        }
    }
    __syncthreads();
    if (a.new_slots) {
        // fused store: a sequence whose context length is rejected gets no item, so no decode warp stores
        // its new row; store it here (one warp per such sequence), as pa_store_kv would
        const int lane = tid & 31;
        const int chunks = a.num_kv_heads * a.head_dim / 8;    // 16-byte pieces of one K (or V) row
        for (int s = tid >> 5; s < a.batch; s += kPlanThreads / 32) {
            if (dec_tiles(a, s, false) > 0) continue;
            const int32_t sl = __ldg(a.new_slots + s);
            if (sl < 0) continue;
            if ((int64_t)sl >= a.num_slots) {
                if (lane == 0) report(a.dev_error, PA_DEVERR_SLOT);
                continue;
            }
            const uint4 *ks = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(a.k_new) +
                                                              (int64_t)s * a.kn_stride);
            const uint4 *vs = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(a.v_new) +
                                                              (int64_t)s * a.vn_stride);
            uint4 *kd = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.k_cache) + (int64_t)sl * chunks * 8);
            uint4 *vd = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.v_cache) + (int64_t)sl * chunks * 8);
            for (int c = lane; c < chunks; c += 32) {
                kd[c] = __ldg(ks + c);
                vd[c] = __ldg(vs + c);
            }
        }
    }
    int4 *items = reinterpret_cast<int4 *>(reinterpret_cast<char *>(a.plan_ws) + kPlanHdrBytes);
    const int npairs = a.batch * a.num_kv_heads;     // < 2^31: the host bounds batch and KV heads
    // whole pairs: one thread each; split pairs go to a list (or, past its capacity, are written here)
    __shared__ int s_split[kPlanSplitList];
    __shared__ int s_nsplit;
    // pairs with no tiles after t_offset whose part_base partials the decode kernel would otherwise fold in
    // (a shared-prefix sequence with no private token): merged here, a warp each
    __shared__ int s_bare[kPlanSplitList];
    __shared__ int s_nbare;
    if (tid == 0) s_nsplit = s_nbare = 0;
    __syncthreads();
    for (int pr = tid; pr < npairs; pr += kPlanThreads) {
        const int s = pr / a.num_kv_heads, kvh = pr - s * a.num_kv_heads;
        const int tiles = s < kPlanCache ? s_tiles[s] : dec_tiles(a, s, false);
        const SplitGeom g = dec_split_geom(tiles, whole, chunk);
        if (a.merge_count) a.merge_count[pr] = g.n;   // splits of the pair still to finish (the decode counts down)
        if (g.n == 0) {
            if (a.merge_count && a.part_base > 0 && tiles == 0 && dec_ctx(a, s) == a.t_offset && a.t_offset > 0) {
                const int bi = atomicAdd(&s_nbare, 1);
                if (bi < kPlanSplitList) s_bare[bi] = pr;
                else plan_merge_bare(a, s, kvh, 0, 1);
            }
            if (pr < n_first) items[pr] = make_int4(kDecSkip, 0, 0, 0);   // CTA pr takes its first item from the counter
            continue;
        }
        const int ctx = s < kPlanCache ? s_ctx[s] : dec_ctx(a, s);
        if (g.n == 1) {
            items[pr < n_first ? pr : atomicAdd(&s_off[bucket(tiles)], 1)] = make_int4(s, kvh, a.t_offset, ctx);
            continue;
        }
        const int li = atomicAdd(&s_nsplit, 1);
        if (li < kPlanSplitList) {
            s_split[li] = pr;
            continue;
        }
        // past the list's capacity: this thread writes the pair's splits, one slot each
        for (int j = 0; j < g.n; ++j) {
            const int b0 = dec_split_begin(g, chunk, j), b1 = dec_split_begin(g, chunk, j + 1);
            items[j == 0 && pr < n_first ? pr : atomicAdd(&s_off[bucket(b1 - b0)], 1)] =
                make_int4(s, kvh | (j << 16), a.t_offset + b0 * kTile, j == g.n - 1 ? ctx : a.t_offset + b1 * kTile);
        }
    }
    __syncthreads();
    // listed split pairs: one warp each, its lanes writing the splits (a long context has dozens)
    const int lane = tid & 31;
    const int nlisted = min(s_nsplit, kPlanSplitList);
    for (int li = tid >> 5; li < nlisted; li += kPlanThreads / 32) {
        const int pr = s_split[li];
        const int s = pr / a.num_kv_heads, kvh = pr - s * a.num_kv_heads;
        const int tiles = s < kPlanCache ? s_tiles[s] : dec_tiles(a, s, false);
        const SplitGeom g = dec_split_geom(tiles, whole, chunk);
        const int ctx = s < kPlanCache ? s_ctx[s] : dec_ctx(a, s);
        const int ct = chunk * kTile;
        // the full chunks take consecutive slots of their bucket (lane 0 reserves them); each tail piece
        // (lanes 0 .. np-1) reserves its own slot; split 0 of a first pair goes to its fixed slot
        const bool first = pr < n_first;
        const int j0 = first && g.nfull > 0 ? 1 : 0;   // full chunks from j0 on are bucketed
        int pos = 0;
        if (lane == 0 && g.nfull > j0) pos = atomicAdd(&s_off[bucket(chunk)], g.nfull - j0);
        pos = __shfl_sync(0xffffffffu, pos, 0);
        for (int j = j0 + lane; j < g.nfull; j += 32)
            items[pos + j - j0] = make_int4(s, kvh | (j << 16), a.t_offset + j * ct, a.t_offset + (j + 1) * ct);
        if (lane == 0 && j0 == 1) items[pr] = make_int4(s, kvh, a.t_offset, a.t_offset + ct);
        if (lane < g.np) {
            const int j = g.nfull + lane;
            const int b0 = dec_split_begin(g, chunk, j), b1 = dec_split_begin(g, chunk, j + 1);
            items[j == 0 && first ? pr : atomicAdd(&s_off[bucket(b1 - b0)], 1)] =
                make_int4(s, kvh | (j << 16), a.t_offset + b0 * kTile, j == g.n - 1 ? ctx : a.t_offset + b1 * kTile);
        }
    }
    const int nbare = min(s_nbare, kPlanSplitList);
    for (int bi = tid >> 5; bi < nbare; bi += kPlanThreads / 32) {
        const int pr = s_bare[bi];
        plan_merge_bare(a, pr / a.num_kv_heads, pr % a.num_kv_heads, lane, 32);
    }
}

struct DecItem {
    int s, kvh, split, t_begin, t_end, ntiles, ctx;
};

// In-kernel merge of a split pair: weights of up to kMergeW (head, split) partials staged in shared memory;
// used when the host plan cuts a pair into at most kMergeMaxSplits splits.
constexpr int kMergeW = 1024;
constexpr int kMergeMaxSplits = 8;
constexpr int kFold = 8;             // earlier partials a pair's only item requests at once

// A consumer-wide vote (the 128 threads of warps 0-3, named barrier 1): true iff v is true for all.
__device__ __forceinline__ bool consumers_all(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, 1, %2, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "n"(kConsumerWarps * 32)
        : "memory");
    return r != 0;
}

// Merge the nsp partials of (sequence s, KV head kvh) -- every split of the pair -- into its G output rows:
// log-sum-exp weights staged in shared memory, then weighted sums of the fp32 partials, four elements per
// thread.  Run by the 128 consumer threads of the CTA that finished the pair's last split; red_o (the merge
// area) is free.
template <int D>
__device__ __forceinline__ void merge_pair(const DecodeArgs &a, int s, int kvh, int nsp, int G, float *red_o,
                                           float *s_w, float *s_wsum) {
    __threadfence();   // (thread 0 acquired the other splits' partials; order this thread's reads after it)
    const int tid = threadIdx.x;
    const int64_t pb0 = ((int64_t)s * a.num_q_heads + (int64_t)kvh * G) * a.part_slots;
    const int64_t orow = dec_row(a, s) * a.num_q_heads + (int64_t)kvh * G;
    if (G * nsp <= kMergeW) {
        // weights exp2(lse_j - max) per head, staged in shared memory, and their sums
        for (int i = tid; i < G * nsp; i += kConsumerWarps * 32) {
            const int g = i / nsp, j = i - g * nsp;
            s_w[i] = __ldcg(a.part_lse + pb0 + (int64_t)g * a.part_slots + j);
        }
        consumer_sync();
        if (tid < G) {
            float m = -INFINITY, sum = 0.f;
            for (int j = 0; j < nsp; ++j) m = fmaxf(m, s_w[tid * nsp + j]);
            for (int j = 0; j < nsp; ++j) {
                const float w = fast_exp2(s_w[tid * nsp + j] - m);
                s_w[tid * nsp + j] = w;
                sum += w;
            }
            s_wsum[tid] = sum;
        }
        consumer_sync();
        // weighted sums over the splits, four elements per thread; with few columns several threads
        // share a column (each a stride of the splits) and their sums meet in the merge area
        const int ncol = G * D / 4;
        const int ngrp = max(1, min(4, kConsumerWarps * 32 / ncol));
        float4 *acc = reinterpret_cast<float4 *>(red_o);   // [ngrp][ncol]
        for (int c = tid; c < ncol * ngrp; c += kConsumerWarps * 32) {
            const int col = c % ncol, grp = c / ncol;
            const int g = col / (D / 4), d4 = col % (D / 4);
            const float4 *src = reinterpret_cast<const float4 *>(a.part_o + (pb0 + (int64_t)g * a.part_slots) * D) + d4;
            float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
            for (int j = grp; j < nsp; j += ngrp) {
                const float w = s_w[g * nsp + j];
                const float4 v = __ldcg(src + (int64_t)j * (D / 4));
                t.x += w * v.x;
                t.y += w * v.y;
                t.z += w * v.z;
                t.w += w * v.w;
            }
            acc[grp * ncol + col] = t;
        }
        consumer_sync();
        for (int col = tid; col < ncol; col += kConsumerWarps * 32) {
            float4 t = acc[col];
            for (int grp = 1; grp < ngrp; ++grp) {
                const float4 u = acc[grp * ncol + col];
                t.x += u.x;
                t.y += u.y;
                t.z += u.z;
                t.w += u.w;
            }
            const int g = col / (D / 4), d4 = col % (D / 4);
            const float inv = 1.f / s_wsum[g];
            uint2 o2;
            o2.x = pack_bf16(t.x * inv, t.y * inv);
            o2.y = pack_bf16(t.z * inv, t.w * inv);
            reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(a.out) + (orow + g) * D)[d4] = o2;
        }
    } else {
        // more (head, split) partials than the staging area holds (a very long context cut into
        // thousands of splits): element by element
        for (int e = tid; e < G * D; e += kConsumerWarps * 32) {
            const int g = e / D, d = e % D;
            const int64_t pb = pb0 + (int64_t)g * a.part_slots;
            float mt = -INFINITY;
            for (int j = 0; j < nsp; ++j) mt = fmaxf(mt, __ldcg(a.part_lse + pb + j));
            float num = 0.f, den = 0.f;
            for (int j = 0; j < nsp; ++j) {
                const float w = fast_exp2(__ldcg(a.part_lse + pb + j) - mt);
                num += w * __ldcg(a.part_o + (pb + j) * D + d);
                den += w;
            }
            static_cast<__nv_bfloat16 *>(a.out)[(orow + g) * D + d] = __float2bfloat16_rn(num / den);
        }
    }
}

// kFused: the pa_store_kv_decode variant (store fused in); a separate instantiation, so the plain decode
// carries none of its registers.
template <int D, bool kFused>
__global__ void __launch_bounds__(kThreads, 2)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const DecodeArgs a) {
    using C = DecodeCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *empty = full + C::kStages;
    uint64_t *qfull = empty + C::kStages;       // [2]
    uint64_t *qempty = qfull + 2;               // [2]
    const int G = a.group;
    float *red_o = reinterpret_cast<float *>(smem + C::red_off(G));   // [warp][G][D]
    float *red_ml = red_o + kConsumerWarps * G * D;                 // [warp][G][2]

    int4 *desc = reinterpret_cast<int4 *>(smem + C::kBarOff + 192);   // [2]: the item of each Q slot
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the combine kernel (launched next, as this grid's programmatic dependent) may be scheduled now: its CTAs
    // only wait (griddepcontrol.wait) for this grid to finish, in resources this one leaves free
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const uint32_t ring = smem_u32(smem);
    const uint32_t qsm = ring + C::kQOff;
    const uint32_t qslot = (uint32_t)(G * D * 2);

    if (threadIdx.x == 0) {
        for (int st = 0; st < C::kStages; ++st) {
            mbar_init(smem_u32(full + st), 1);
            mbar_init(smem_u32(empty + st), kConsumerWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(qfull + i), 1);
            mbar_init(smem_u32(qempty + i), kConsumerWarps);
        }
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------ producer --
        // CTA c < n_first owns the first split of pair c.  For a batch of up to kDecLocalCut sequences the warp
        // sums the call's work itself and cuts the pair as the planning kernel does (dec_cut on the same
        // total), so the first item -- its Q rows, all its tiles, the consumers' work on them -- runs while
        // the planning kernel's table is still being written; only the next item waits for the table.
        const int n_first = min((int)gridDim.x, a.batch * a.num_kv_heads);
        int4 d_first = make_int4(-1, 0, 0, 0);   // the item the planning kernel writes into slot c, or none
        if ((int)blockIdx.x < n_first && a.batch <= kDecLocalCut) {
            int whole, chunk;
            dec_cut(a, dec_total_warp(a, lane), (int)gridDim.x, whole, chunk);
            const int s0 = blockIdx.x / a.num_kv_heads, kvh0 = blockIdx.x % a.num_kv_heads;
            const SplitGeom g = dec_split_geom(dec_tiles(a, s0, false), whole, chunk);
            if (g.n > 0)   // {s, kvh, t_offset, end of the first split}
                d_first = make_int4(s0, kvh0, a.t_offset,
                                    g.n == 1 ? dec_ctx(a, s0) : a.t_offset + dec_split_begin(g, chunk, 1) * kTile);
        }
        // One thread.  The next item's index is taken when three tiles of the current item remain to be
        // issued (not earlier: an item taken early is held back from idle CTAs) and its record is read a tile
        // later, so both latencies run under the copies already in the ring.  (Reading each tile's block ids
        // a tile ahead measured slower than reading them just before the copy.)
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            const int B = a.block_size, box = a.box_tokens;
            uint32_t gt = 0, nqi = 0;             // tiles and Q copies issued so far
            bool ok = true;
            const uint32_t qbytes = (uint32_t)(G * D * 2);
            auto q_rows = [&](int s, int kvh) {   // Q rows of the GQA group: one contiguous bulk copy
                return static_cast<const __nv_bfloat16 *>(a.q) + (dec_row(a, s) * a.num_q_heads + (int64_t)kvh * G) * D;
            };
            // the copies of one tile (tokens tile0 .. min(tile0 + kTile, t_end) - 1) into stage st
            auto load_tile = [&](const int32_t *bt, int kvh, int tile0, int t_end, int st) {
                const int nbox = (min(kTile, t_end - tile0) + box - 1) / box;
                const uint32_t fb = smem_u32(full + st);
                mbar_arrive_expect_tx(fb, (uint32_t)(nbox * box * 128 * C::kHalves * 2));
                const uint32_t kdst = ring + st * C::kStageBytes;
                const uint32_t vdst = kdst + C::kKvBytes;
                for (int b = 0; b < nbox; ++b) {
                    const int tok = tile0 + b * box;
                    const int blk = __ldg(bt + tok / B);
                    int row;
                    if ((unsigned)blk < (unsigned)a.num_blocks) {
                        row = blk * B + (tok % B);
                    } else {               // out-of-range id: load zeros instead (TMA fills)
                        report(a.dev_error, PA_DEVERR_BLOCK_ID);
                        row = -box;
                    }
#pragma unroll
                    for (int h = 0; h < C::kHalves; ++h) {
                        const uint32_t off = h * kHalfBytes + b * box * 128;
                        tma_load_3d(kdst + off, &tm_k, h * 64, kvh, row, fb);
                        tma_load_3d(vdst + off, &tm_v, h * 64, kvh, row, fb);
                    }
                }
            };
            DecPlanHdr *hdr = reinterpret_cast<DecPlanHdr *>(a.plan_ws);
            const int4 *items = reinterpret_cast<const int4 *>(reinterpret_cast<const char *>(a.plan_ws) + kPlanHdrBytes);
            const int4 kEnd = make_int4(-1, 0, 0, 0);
            int n_items = 0;
            bool waited = false;
            auto wait_table = [&]() {   // the planning kernel's table is complete
                if (waited) return;
                asm volatile("griddepcontrol.wait;" ::: "memory");
                n_items = __ldcg(&hdr->n_items);
                waited = true;
            };
            int4 d = d_first;
            int idx = 0;
            if (d.x < 0) {
                // the first item is this CTA's own slot (if it has one); the rest come from the counter
                wait_table();
                idx = (int)blockIdx.x < n_first ? (int)blockIdx.x : atomicAdd(&hdr->counter, 1);
                d = idx < n_items ? __ldcg(items + idx) : kEnd;
            }
            while (ok) {
                const int qs = nqi & 1;
                if (nqi >= 2 && !mbar_wait(smem_u32(qempty + qs), ((nqi >> 1) - 1) & 1, a.dev_error)) break;
                if (d.x == kDecSkip) {            // a first slot whose pair has no work
                    wait_table();
                    idx = atomicAdd(&hdr->counter, 1);
                    d = idx < n_items ? __ldcg(items + idx) : kEnd;
                    continue;
                }
                if (d.x < 0) {                    // end of the stream: an item with s < 0, no copy
                    desc[qs] = d;
                    mbar_arrive(smem_u32(qfull + qs));
                    ++nqi;
                    break;
                }
                int idx_next = n_items;
                int4 d_next = kEnd;
                desc[qs] = d;                     // the item rides in the Q slot's descriptor
                const int s = d.x, kvh = d.y & 0xffff, t_begin = d.z, t_end = d.w;
                const int ntiles = (t_end - t_begin + kTile - 1) / kTile;
                mbar_arrive_expect_tx(smem_u32(qfull + qs), qbytes);
                bulk_load(qsm + qs * qslot, q_rows(s, kvh), qbytes, smem_u32(qfull + qs));
                ++nqi;
                const int32_t *bt = a.block_table + (int64_t)s * a.bt_stride;
                for (int t = 0; t < ntiles; ++t, ++gt) {
                    const int st = gt % C::kStages;
                    if (gt >= (uint32_t)C::kStages &&
                        !mbar_wait(smem_u32(empty + st), ((gt / C::kStages) & 1) ^ 1, a.dev_error)) {
                        ok = false;
                        break;
                    }
                    load_tile(bt, kvh, t_begin + t * kTile, t_end, st);
                    // the next item: index and record, issued now and used when this item's copies are out
                    if (t == max(0, ntiles - 3)) {
                        wait_table();
                        idx_next = atomicAdd(&hdr->counter, 1);
                    }
                    if (t == max(0, ntiles - 2)) d_next = idx_next < n_items ? __ldcg(items + idx_next) : kEnd;
                }
                d = d_next;
            }
            // leave no copy in flight: wait (bounded) for the last load of every stage and the last Q copies
            // (the end marker's slot completes by its plain arrive); on the normal path the consumers have
            // already waited for them all and these return at once
            for (uint32_t i = (gt > (uint32_t)C::kStages ? gt - C::kStages : 0); i < gt; ++i)
                mbar_wait(smem_u32(full + i % C::kStages), (i / C::kStages) & 1, a.dev_error);
            for (uint32_t i = (nqi > 2 ? nqi - 2 : 0); i < nqi; ++i)
                mbar_wait(smem_u32(qfull + (i & 1)), (i >> 1) & 1, a.dev_error);
        }
        return;
    }

    // ---------------------------------------------------------- consumers --
    const int g0 = lane >> 2;             // accumulator rows g0 and g0 + 8
    const int c2 = (lane & 3) * 2;        // accumulator columns c2, c2 + 1
    const int mi = lane >> 3, mr = lane & 7;  // ldmatrix: matrix index / row this lane addresses
    uint32_t gt = 0, nqi = 0;
    bool ok = true;
    // In-kernel merge (a.merge_count): thread 0 counts a finished split down with an atomic whose result it
    // looks at only one item later (or when the stream ends), so no consumer waits for the round trip; if the
    // count reached zero this CTA finished the pair's last split and merges the pair (flush_pending).
    int pend_left = 0, hdr_whole = -1, hdr_chunk = 0;
    int4 pend = make_int4(0, 0, 0, 0);   // s, kvh, ctx, counted
    __shared__ int4 s_pend;
    __shared__ float s_w[kMergeW], s_wsum[16];
    auto flush_pending = [&]() {
        if (threadIdx.x == 0) {
            int nsp = 0;
            if (pend.w && pend_left == 1) {
                if (hdr_whole < 0) {
                    const DecPlanHdr *hdr = reinterpret_cast<const DecPlanHdr *>(a.plan_ws);
                    hdr_whole = __ldcg(&hdr->whole);
                    hdr_chunk = __ldcg(&hdr->chunk);
                }
                nsp = dec_nsplit((pend.z - a.t_offset + kTile - 1) / kTile, hdr_whole, hdr_chunk);
            }
            s_pend = make_int4(pend.x, pend.y, nsp, 0);
            pend.w = 0;
        }
        consumer_sync();
        const int4 pm = s_pend;
        if (pm.z > 0) merge_pair<D>(a, pm.x, pm.y, a.part_base + pm.z, G, red_o, s_w, s_wsum);
        consumer_sync();   // s_pend and the merge area are free again
    };
    for (;;) {
        // the next item, from the producer; the consumers leave together at the end marker or after a
        // timed-out wait (a wait that gave up leaves the results garbage and dev_error says so)
        const int qs = nqi & 1;
        const bool landed = ok && mbar_wait(smem_u32(qfull + qs), (nqi >> 1) & 1, a.dev_error);
        const int4 d = desc[qs];
        if (!consumers_all(landed && d.x >= 0)) break;
        DecItem it;
        it.s = d.x;
        it.kvh = d.y & 0xffff;
        it.split = d.y >> 16;
        it.t_begin = d.z;
        it.t_end = d.w;
        it.ntiles = (it.t_end - it.t_begin + kTile - 1) / kTile;
        it.ctx = dec_ctx(a, it.s);
        // fused store: this warp owns the new token's row if position ctx - 1 falls in its slice of the
        // pair's last split; the row is staged now and used when its tile lands
        // own: 0, or 1 (this warp stores the new row) | 2 (the slot is the row this decode reads: the tile is
        // patched too); the tile and row of the new token follow from ctx - 1 - t_begin
        int own = 0;
        if (kFused && it.t_end == it.ctx && ((it.ctx - 1 - it.t_begin) % kTile) / 16 == warp) {
            const int32_t sl = __ldg(a.new_slots + it.s);
            if (sl >= 0) {
                const int p = it.ctx - 1;
                const int32_t blk = __ldg(a.block_table + (int64_t)it.s * a.bt_stride + p / a.block_size);
                const int64_t expect = (int64_t)blk * a.block_size + p % a.block_size;
                if ((int64_t)sl >= a.num_slots) {
                    if (lane == 0) report(a.dev_error, PA_DEVERR_SLOT);
                } else {
                    // a slot other than the row this decode reads is still written (as pa_store_kv would)
                    if (sl != expect && lane == 0) report(a.dev_error, PA_DEVERR_SLOT);
                    own = sl == expect ? 3 : 1;
                    // lane c < D/8 copies 16 bytes of K, lane D/8 + c those of V, into the staging row
                    // (asynchronously: the latency hides behind the item's earlier tiles)
                    if (lane < D / 4) {
                        const bool isv = lane >= D / 8;
                        const int c = isv ? lane - D / 8 : lane;
                        const __nv_bfloat16 *src =
                            static_cast<const __nv_bfloat16 *>(isv ? a.v_new : a.k_new) +
                            (int64_t)it.s * (isv ? a.vn_stride : a.kn_stride) + (int64_t)it.kvh * D + c * 8;
                        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(ring + C::kNewOff + lane * 16),
                                     "l"(src)
                                     : "memory");
                    }
                    asm volatile("cp.async.commit_group;" ::: "memory");
                }
            }
        }
        // Q fragments; rows past the group are zero
        ++nqi;
        uint32_t qa[D / 16][4];
        {
            const uint32_t qb = qsm + qs * qslot;
            const bool r0 = g0 < G, r1 = g0 + 8 < G;
            const uint32_t a0 = qb + (r0 ? g0 : 0) * D * 2, a1 = qb + (r1 ? g0 + 8 : 0) * D * 2;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t k0 = (ks * 16 + c2) * 2;
                uint32_t v0, v1, v2, v3;
                asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v0) : "r"(a0 + k0));
                asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v1) : "r"(a1 + k0));
                asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v2) : "r"(a0 + k0 + 16));
                asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v3) : "r"(a1 + k0 + 16));
                qa[ks][0] = r0 ? v0 : 0u;
                qa[ks][1] = r1 ? v1 : 0u;
                qa[ks][2] = r0 ? v2 : 0u;
                qa[ks][3] = r1 ? v3 : 0u;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(qempty + qs));

        float m_run[2] = {-INFINITY, -INFINITY};
        float l_run[2] = {0.f, 0.f};
        float o[D / 8][4];
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;

        for (int t = 0; t < it.ntiles; ++t, ++gt) {
            const int st = gt % C::kStages;
            const bool landed = ok && mbar_wait(smem_u32(full + st), (gt / C::kStages) & 1, a.dev_error);
            if (!__all_sync(0xffffffffu, landed)) ok = false;
            const uint32_t kbase = ring + st * C::kStageBytes;
            const uint32_t vbase = kbase + C::kKvBytes;
            const int tok0 = it.t_begin + t * kTile + warp * 16;   // first token of this warp's slice
            const bool own_tile = kFused && own != 0 && t == (it.ctx - 1 - it.t_begin) / kTile;   // warp-uniform
            if (own_tile) {
                asm volatile("cp.async.wait_all;" ::: "memory");   // this lane's staged 16 bytes
                if (lane < D / 4) {
                    const bool isv = lane >= D / 8;
                    const uint32_t c = isv ? lane - D / 8 : lane;
                    uint4 nrow;
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(nrow.x), "=r"(nrow.y), "=r"(nrow.z), "=r"(nrow.w)
                                 : "r"(ring + C::kNewOff + lane * 16)
                                 : "memory");
                    if (own & 2) {
                        const uint32_t dst =
                            (isv ? vbase : kbase) + (c >> 3) * kHalfBytes + swz128((uint32_t)((it.ctx - 1 - it.t_begin) % kTile), c & 7);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(nrow.x),
                                     "r"(nrow.y), "r"(nrow.z), "r"(nrow.w)
                                     : "memory");
                    }
                    __nv_bfloat16 *dstg = static_cast<__nv_bfloat16 *>(isv ? a.v_cache : a.k_cache) +
                                          ((int64_t)__ldg(a.new_slots + it.s) * a.num_kv_heads + it.kvh) * D + c * 8;
                    *reinterpret_cast<uint4 *>(dstg) = nrow;
                }
                __syncwarp();
            }

            // S = Q K^T over this warp's 16 tokens (two n-tiles of 8 tokens)
            float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const int trow = warp * 16 + (mi >> 1) * 8 + mr;
                const int dch = ks * 2 + (mi & 1);
                uint32_t b0n0, b1n0, b0n1, b1n1;
                ldmatrix_x4(kbase + (dch >> 3) * kHalfBytes + swz128(trow, dch & 7), b0n0, b1n0, b0n1, b1n1);
                mma_bf16_16816(sc[0], qa[ks], b0n0, b1n0);
                mma_bf16_16816(sc[1], qa[ks], b0n1, b1n1);
            }

            // scale into log2 units and select out positions past the end
            const bool partial = tok0 + 16 > it.t_end;
#pragma unroll
            for (int n = 0; n < 2; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int tok = tok0 + n * 8 + c2 + (e & 1);
                    const float v = sc[n][e] * a.scale_log2;
                    sc[n][e] = (!partial || tok < it.t_end) ? v : -INFINITY;
                }

            // online softmax (rows g0 and g0 + 8)
            float mx[2];
            mx[0] = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
            mx[1] = fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3]));
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
                mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
            }
            float corr[2], ref[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const float m_new = fmaxf(m_run[r], mx[r]);
                ref[r] = m_new == -INFINITY ? 0.f : m_new;
                corr[r] = fast_exp2(m_run[r] - ref[r]);
                m_run[r] = m_new;
            }
            float p[2][4];
#pragma unroll
            for (int n = 0; n < 2; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) p[n][e] = fast_exp2(sc[n][e] - ref[e >> 1]);
            l_run[0] = l_run[0] * corr[0] + (p[0][0] + p[0][1] + p[1][0] + p[1][1]);
            l_run[1] = l_run[1] * corr[1] + (p[0][2] + p[0][3] + p[1][2] + p[1][3]);
            if (!__all_sync(0xffffffffu, corr[0] == 1.f && corr[1] == 1.f)) {
#pragma unroll
                for (int nt = 0; nt < D / 8; ++nt) {
                    o[nt][0] *= corr[0];
                    o[nt][1] *= corr[0];
                    o[nt][2] *= corr[1];
                    o[nt][3] *= corr[1];
                }
            }
            uint32_t pa[4];
            pa[0] = pack_bf16(p[0][0], p[0][1]);
            pa[1] = pack_bf16(p[0][2], p[0][3]);
            pa[2] = pack_bf16(p[1][0], p[1][1]);
            pa[3] = pack_bf16(p[1][2], p[1][3]);

            // V fragments hold tokens tok0 + c2 + {0,1} (b0) and tok0 + 8 + c2 + {0,1} (b1)
            uint32_t vm0 = 0xffffffffu, vm1 = 0xffffffffu;
            if (partial) {
                vm0 = (tok0 + c2 < it.t_end ? 0x0000ffffu : 0u) | (tok0 + c2 + 1 < it.t_end ? 0xffff0000u : 0u);
                vm1 = (tok0 + 8 + c2 < it.t_end ? 0x0000ffffu : 0u) | (tok0 + 9 + c2 < it.t_end ? 0xffff0000u : 0u);
            }
#pragma unroll
            for (int jp = 0; jp < D / 16; ++jp) {
                const int trow = warp * 16 + (mi & 1) * 8 + mr;
                const int dch = jp * 2 + (mi >> 1);
                uint32_t b0a, b1a, b0b, b1b;
                ldmatrix_x4_trans(vbase + (dch >> 3) * kHalfBytes + swz128(trow, dch & 7), b0a, b1a, b0b, b1b);
                b0a &= vm0;
                b1a &= vm1;
                b0b &= vm0;
                b1b &= vm1;
                mma_bf16_16816(o[2 * jp], pa, b0a, b1a);
                mma_bf16_16816(o[2 * jp + 1], pa, b0b, b1b);
            }
            // a patched stage is rewritten by a later TMA load: order the generic writes before it
            if (own_tile && (own & 2)) fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(empty + st));
        }

#pragma unroll
        for (int r = 0; r < 2; ++r) {
            l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
            l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
        }
        // ------------------------------------------ merge the four warps --
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int g = g0 + r * 8;
            if (g < G) {
                float *dst = red_o + (warp * G + g) * D;
#pragma unroll
                for (int nt = 0; nt < D / 8; ++nt) {
                    dst[nt * 8 + c2] = o[nt][2 * r];
                    dst[nt * 8 + c2 + 1] = o[nt][2 * r + 1];
                }
                if ((lane & 3) == 0) {
                    red_ml[(warp * G + g) * 2] = m_run[r];
                    red_ml[(warp * G + g) * 2 + 1] = l_run[r];
                }
            }
        }
        consumer_sync();
        // the pair's only item: write the result directly -- merged with the part_base partials written before
        // this launch (shared-prefix chunks) when there are some and this kernel merges
        const bool only = it.t_begin == a.t_offset && it.t_end == it.ctx;
        const bool direct = only && (a.part_base == 0 || a.merge_count);
        for (int e = threadIdx.x; e < G * D; e += kConsumerWarps * 32) {
            const int g = e / D, d = e % D;
            float mt = -INFINITY;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) mt = fmaxf(mt, red_ml[(w * G + g) * 2]);
            float lt = 0.f, ot = 0.f;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) {
                const float mw = red_ml[(w * G + g) * 2];
                const float f = mw == -INFINITY ? 0.f : fast_exp2(mw - mt);
                lt += f * red_ml[(w * G + g) * 2 + 1];
                ot += f * red_o[(w * G + g) * D + d];
            }
            const int h = it.kvh * G + g;
            if (direct && a.part_base > 0) {
                // fold in the earlier partials of (s, h): log-sum-exp weights against this item's own.  The
                // partials are requested kFold at a time, all before the first is used (one round trip each).
                const int64_t pb = ((int64_t)it.s * a.num_q_heads + h) * a.part_slots;
                const float lse_self = mt + __log2f(lt);
                float m = lse_self, num = 0.f, den = 0.f, own = ot / lt;
                for (int j0 = 0; j0 < a.part_base; j0 += kFold) {
                    float pl[kFold], po[kFold];
#pragma unroll
                    for (int j = 0; j < kFold; ++j) {
                        const bool in = j0 + j < a.part_base;
                        pl[j] = in ? __ldcg(a.part_lse + pb + j0 + j) : -INFINITY;
                        po[j] = in ? __ldcg(a.part_o + (pb + j0 + j) * D + d) : 0.f;
                    }
                    float mb = m;
#pragma unroll
                    for (int j = 0; j < kFold; ++j) mb = fmaxf(mb, pl[j]);
                    const float c = fast_exp2(m - mb);   // rescale what was summed so far
                    num *= c;
                    den *= c;
                    m = mb;
#pragma unroll
                    for (int j = 0; j < kFold; ++j) {
                        const float w = fast_exp2(pl[j] - m);
                        num += w * po[j];
                        den += w;
                    }
                }
                const float ws = fast_exp2(lse_self - m);
                static_cast<__nv_bfloat16 *>(a.out)[(dec_row(a, it.s) * a.num_q_heads + h) * D + d] =
                    __float2bfloat16_rn((num + ws * own) / (den + ws));
            } else if (direct) {
                static_cast<__nv_bfloat16 *>(a.out)[(dec_row(a, it.s) * a.num_q_heads + h) * D + d] =
                    __float2bfloat16_rn(ot / lt);
            } else {
                const int64_t pi = ((int64_t)it.s * a.num_q_heads + h) * a.part_slots + a.part_base + it.split;
                a.part_o[pi * D + d] = ot / lt;
                if (d == 0) a.part_lse[pi] = mt + __log2f(lt);
            }
        }
        if (a.merge_count) {
            flush_pending();   // the split counted down one item ago (its atomic has long returned)
            if (!direct) {
                // this split is finished: count it down (release: every consumer's partial stores, ordered
                // before thread 0 by the barrier, are visible before the count; acquire for the last one,
                // which merges)
                if (threadIdx.x == 0) {
                    pend_left = atomic_add_acq_rel(a.merge_count + (int64_t)it.s * a.num_kv_heads + it.kvh, -1);
                    pend = make_int4(it.s, it.kvh, it.ctx, 1);
                }
            }
        }
        consumer_sync();   // the merge area is free for the next item
    }
    if (a.merge_count) flush_pending();   // the last split this CTA counted down
}

// Merge the per-split partials of one (sequence, q-head) by log-sum-exp.  kGroups x D threads: thread
// (g, d) owns output element d for the partial slots g, g + kGroups, ...  The merge is a chain of dependent
// reads, so it is kept short: the context length (an input of the call) is read before the wait for the
// split kernel; after it, the planning header, the log-sum-exps and -- in the wide form (kGroups = 4, used
// when few pairs have many partials: long contexts), for the slot count the host sized -- the first kPre
// partial elements of every thread are all requested at once, and the slots past this pair's count are
// selected out afterwards.  The narrow form requests its partials only once the header says the pair was
// split: with many short CTAs, most of them for pairs that were not split, a request for nothing costs a
// round trip to memory no call wrote in every wave of CTAs.  The kGroups sums are added in shared memory.
constexpr int kLseCache = 1024;

template <int D, int kGroups>
__global__ void __launch_bounds__(D * kGroups) decode_combine_kernel(const DecodeArgs a) {
    constexpr int kPre = kGroups > 1 ? 16 : 4;     // partial elements per thread requested with the header
    const int h = blockIdx.x % a.num_q_heads;
    const int s = blockIdx.x / a.num_q_heads;
    const int ctx = dec_ctx(a, s);              // -1: not this call's work
    asm volatile("griddepcontrol.wait;" ::: "memory");   // partials of the split kernel are visible
    if (ctx < 1 || ctx > a.max_context_len || (int64_t)ctx > (int64_t)a.bt_stride * a.block_size ||
        ctx < a.t_offset)
        return;
    // partials: part_base slots written before this launch (shared-prefix chunks), then the splits, cut as
    // the planning kernel cut them; a pair of one split and nothing else was written directly
    const DecPlanHdr *hdr = reinterpret_cast<const DecPlanHdr *>(a.plan_ws);
    const int64_t base = ((int64_t)s * a.num_q_heads + h) * a.part_slots;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int g = tid / D, d = tid % D;
    const int nmax = a.part_slots;              // slots of this pair: an upper bound of its partial count
    const float *lse = a.part_lse + base;
    const float *po = a.part_o + base * D + d;
    const int whole = __ldcg(&hdr->whole), chunk = __ldcg(&hdr->chunk);
    float l0 = tid < nmax ? __ldcg(lse + tid) : -INFINITY;
    float pv[kPre];
    if (kGroups > 1) {
#pragma unroll
        for (int i = 0; i < kPre; ++i) {
            const int k = g + i * kGroups;
            pv[i] = k < nmax ? __ldcg(po + (int64_t)k * D) : 0.f;
        }
    }
    const int nsplit = dec_nsplit((ctx - a.t_offset + kTile - 1) / kTile, whole, chunk);
    if (a.part_base == 0 && nsplit <= 1) return;
    const int n = a.part_base + nsplit;
    if (kGroups == 1) {
#pragma unroll
        for (int i = 0; i < kPre; ++i) pv[i] = i < n ? __ldcg(po + (int64_t)i * D) : 0.f;
    }
    constexpr int kWarps = D * kGroups / 32;
    __shared__ float s_lse[kLseCache];
    __shared__ float s_red[kWarps];
    __shared__ float s_num[kGroups][D];
    __shared__ float s_den[kGroups];
    // 1. the largest log-sum-exp
    float mx = -INFINITY;
    for (int k = tid; k < n; k += D * kGroups) {
        const float l = k == tid ? l0 : lse[k];
        if (k < kLseCache) s_lse[k] = l;
        mx = fmaxf(mx, l);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) s_red[wid] = mx;
    __syncthreads();
    float mt = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) mt = fmaxf(mt, s_red[w]);
    // 2. this thread's share of the weighted sum (slots past n are selected out, never multiplied)
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int i = 0; i < kPre; ++i) {
        const int k = g + i * kGroups;
        if (k < n) {
            const float l = k < kLseCache ? s_lse[k] : lse[k];
            const float w = l == -INFINITY ? 0.f : fast_exp2(l - mt);
            den += w;
            num += w * pv[i];
        }
    }
#pragma unroll 8
    for (int k = g + kPre * kGroups; k < n; k += kGroups) {
        const float l = k < kLseCache ? s_lse[k] : lse[k];
        const float w = l == -INFINITY ? 0.f : fast_exp2(l - mt);
        den += w;
        num += w * po[(int64_t)k * D];
    }
    if (kGroups > 1) {
        s_num[g][d] = num;
        if (d == 0) s_den[g] = den;
        __syncthreads();
        if (g != 0) return;
#pragma unroll
        for (int q = 1; q < kGroups; ++q) {
            num += s_num[q][d];
            den += s_den[q];
        }
    }
    static_cast<__nv_bfloat16 *>(a.out)[(dec_row(a, s) * a.num_q_heads + h) * D + d] = __float2bfloat16_rn(num / den);
}

template <int D>
cudaError_t launch_decode_d(const DecodeArgs &a, const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                            cudaStream_t stream) {
    using C = DecodeCfg<D>;
    const bool fused = a.new_slots != nullptr;
    auto kernel = fused ? decode_split_kernel<D, true> : decode_split_kernel<D, false>;
    // attribute and occupancy per (device, variant, G); G <= 16
    static std::atomic<int> resident[64][2][17];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const size_t smem = C::smem_bytes(a.group);
    int per_sm = resident[dev & 63][fused][a.group].load(std::memory_order_acquire);
    if (per_sm == 0) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::smem_bytes(16));
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, smem);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) per_sm = 1;
        resident[dev & 63][fused][a.group].store(per_sm, std::memory_order_release);
    }
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int64_t n_items = (int64_t)a.plan.max_splits * a.batch * a.num_kv_heads;   // an upper bound
    const int64_t slots = (int64_t)per_sm * sms;
    const int grid = (int)(n_items < slots ? n_items : slots);

    // 1. the item table; 2. the persistent decode, launched as its programmatic dependent so that its
    // set-up overlaps the planning (its producer waits for the table with griddepcontrol.wait);
    // 3. the combine, only when partials come from elsewhere too (the split kernel merges its own)
    decode_plan_kernel<<<1, kPlanThreads, 0, stream>>>(a, grid);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kernel, tm_k, tm_v, a);
    if (e != cudaSuccess || (a.plan.max_splits == 1 && a.part_base == 0) || a.merge_count) return e;

    // a few partials per pair, or so many pairs that four threads per element would not fit the GPU at
    // once (a large batch): one thread per element; many partials for few pairs (long contexts): four
    // threads per element, each loading a quarter of them
    const int64_t wide_threads = (int64_t)a.batch * a.num_q_heads * 4 * D;
    const bool wide = a.part_base + a.plan.max_splits > 8 && wide_threads <= (int64_t)sms * 1024;
    cfg.gridDim = dim3((unsigned)(a.batch * a.num_q_heads));
    cfg.blockDim = dim3(wide ? 4 * D : D);
    cfg.dynamicSmemBytes = 0;
    return wide ? cudaLaunchKernelEx(&cfg, decode_combine_kernel<D, 4>, a)
                : cudaLaunchKernelEx(&cfg, decode_combine_kernel<D, 1>, a);
}

}  // namespace

DecodePlan plan_decode(int32_t batch, int32_t num_kv_heads, int32_t max_context_len, int32_t num_splits,
                       int32_t num_sms) {
    DecodePlan p;
    const int64_t full = ((int64_t)max_context_len + kTile - 1) / kTile * kTile;
    int64_t chunk;
    if (num_splits > 0) {
        chunk = ((int64_t)max_context_len + num_splits - 1) / num_splits;
        chunk = (chunk + kTile - 1) / kTile * kTile;
    } else {
        // aim at about eight waves of two CTAs per SM over the whole batch, but
        // never fewer than four tiles per CTA
        const int64_t target = (int64_t)(num_sms > 0 ? num_sms : 148) * 2 * 8;
        const int64_t pairs = (int64_t)batch * num_kv_heads;
        chunk = ((int64_t)max_context_len * pairs + target - 1) / target;
        chunk = (chunk + kTile - 1) / kTile * kTile;
        if (chunk < 4 * kTile) chunk = 4 * kTile;
    }
    if (chunk > full) chunk = full;
    if (chunk < kTile) chunk = kTile;
    p.chunk = (int32_t)chunk;
    p.max_splits = (int32_t)((max_context_len + chunk - 1) / chunk);
    if (p.max_splits < 1) p.max_splits = 1;
    // the planning kernel cuts the last two chunks of a split pair into up to kTailPieces pieces
    if (num_splits <= 0 && p.max_splits >= 2) p.max_splits += kTailPieces - 2;
    p.fixed = num_splits > 0;
    return p;
}

// Planning area: header, item table, then one merge counter per (sequence, KV head).
static size_t decode_counter_offset(const DecodePlan &plan, int32_t batch, int32_t num_kv_heads) {
    const size_t items = (size_t)batch * num_kv_heads * (plan.max_splits > 0 ? plan.max_splits : 1);
    return kPlanHdrBytes + items * sizeof(int4);
}

size_t decode_plan_bytes(const DecodePlan &plan, int32_t batch, int32_t num_kv_heads) {
    const size_t counters = (size_t)batch * num_kv_heads * sizeof(int32_t);
    return (decode_counter_offset(plan, batch, num_kv_heads) + counters + 255) / 256 * 256;
}

DecodeWorkspace decode_workspace_layout(const DecodePlan &plan, int32_t batch, int32_t num_q_heads,
                                        int32_t num_kv_heads, int32_t head_dim, int32_t extra_slots) {
    auto r256 = [](size_t x) { return (x + 255) / 256 * 256; };
    DecodeWorkspace w;
    w.plan_off = 0;
    w.o_off = w.lse_off = w.total = decode_plan_bytes(plan, batch, num_kv_heads);
    if (plan.max_splits <= 1 && extra_slots == 0) return w;
    const size_t n = (size_t)batch * num_q_heads * (plan.max_splits + extra_slots);
    w.lse_off = w.o_off + r256(n * head_dim * sizeof(float));
    w.total = w.lse_off + r256(n * sizeof(float));
    return w;
}

cudaError_t launch_decode(const DecodeArgs &args, const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                          cudaStream_t stream) {
    DecodeArgs a = args;
    // Partials are merged in the split kernel when a pair has only a few splits: a pair's only item folds the
    // part_base partials written before this launch (shared-prefix chunks) into its result, and the CTA that
    // finishes a split pair's last split merges them all.  That saves the combine launch, and each merge is
    // short.  With many splits per pair (long contexts) the pairs' last splits finish together at the end of
    // the grid, and a CTA per pair merging dozens of partials makes a longer tail than the combine kernel,
    // which spreads the merge over many CTAs (measured: 4 splits per pair, -2 us; 32, +10 us).
    a.merge_count = (a.plan.max_splits > 1 || a.part_base > 0) && a.plan.max_splits <= kMergeMaxSplits
                        ? reinterpret_cast<int32_t *>(static_cast<char *>(a.plan_ws) +
                                                      decode_counter_offset(a.plan, a.batch, a.num_kv_heads))
                        : nullptr;
    if (a.head_dim == 128) return launch_decode_d<128>(a, tm_k, tm_v, stream);
    return launch_decode_d<64>(a, tm_k, tm_v, stream);
}

}  // namespace pa
