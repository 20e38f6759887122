// Varlen causal prefill over the paged cache on the 5th-generation tensor
// cores (tcgen05 + TMEM), fed by TMA.
//
// What it computes: for sequence s with n_new query tokens and n_k keys
// (c = n_k - n_new cached keys before them), new token i at absolute position
// c + i and q-head h:
//     out[cu_q[s] + i, h] = softmax_j(scale * q . K_j) V_j,  j = 0 .. c + i
// (all n_k keys when not causal): the attention formula of the chenxutan.com
// Nano-vLLM article (section 1.2) evaluated for the uncached segment only,
// with causal alignment to the end of the key range and K/V read through the
// block table -- the flash_attn_varlen_func call of the nano-vllm walkthrough
// (xingyun3d.csdn.net, sections seven and eight).
//
// How:
//  * a Q tile is 128 MMA rows = (128 / G) consecutive new tokens x the G
//    q-heads of one KV head (GQA packing), so one K/V tile feeds all G heads;
//  * a work unit is two adjacent Q tiles (A, then B) of one (sequence, KV
//    head); a one-CTA planning kernel writes the units into a table ordered by
//    decreasing cost (last tiles of every sequence first), and persistent CTAs,
//    one per SM, take them with an atomic counter;
//  * warp 11 (Q): per unit, both Q tiles (3-D tensor map over q) into the Q
//    buffer once the previous unit's S products have read it; warp 8 (K/V):
//    the K and V tiles of 128 keys, gathered block by block through
//    block_table, into a ring of shared-memory slots guarded by mbarriers,
//    running ahead into the next units so that a unit starts on loaded tiles;
//  * warp 9 (MMA): one thread issues tcgen05.mma.cta_group::1.kind::f16 in the
//    order S_A(0) S_B(0) | PV_A(j) S_A(j+1) PV_B(j) S_B(j+1) | ..., so the
//    tensor cores work on one tile while the other tile's softmax runs.
//    TMEM holds S_A, O_A, S_B, O_B (128 columns each); tcgen05.commit signals
//    the mbarriers;
//  * warps 0-3 / 4-7 (softmax of tile A / B): thread t owns TMEM lane t, i.e.
//    one Q row; it reads its S row with tcgen05.ld, selects masked keys out
//    (-inf), keeps a running max in log2 units and rescales O (tcgen05.ld/st)
//    only when the max grew by more than 8 (2^8), writes P as packed bf16
//    back into TMEM over the first columns of its S row (the PV product reads
//    its A operand from TMEM), and after the last key tile divides O by the
//    row sum and stores bf16 rows;
//  * warp 10 (V fix) zeroes the V rows of a unit's last key tile beyond its
//    key range in shared memory before the PV products, so stale or poisoned
//    cache contents never meet a zero weight (0 * NaN is never formed); in the
//    fused-store form it also copies the unit's new K/V rows to their slots.
#include <atomic>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

#include "prefill_common.cuh"

// kFused: the store fused in (pa_store_kv_prefill_varlen) needs a staging area for the rows it copies; at
// D = 128 it takes the room of one K/V ring slot.
template <int D, bool kFused = false>
struct PrefillCfg {
    static constexpr int kHalves = D / 64;
    static constexpr int kSlots = D == 128 ? (kFused ? 4 : 5) : 8;   // K/V ring slots (one K or V tile each)
    static constexpr int kTileBytes = kHalves * kSlab;          // a Q tile, or a K or V tile of 128 keys
    static constexpr int kQOff = 0;                             // Q_A, Q_B
    static constexpr int kRingOff = kQOff + 2 * kTileBytes;
    static constexpr int kStageTokens = 64;                     // fused store: rows per copy round
    static constexpr int kStageOff = kRingOff + kSlots * kTileBytes;   // [token][K row, V row]
    static constexpr int kStageBytes = kFused ? kStageTokens * 4 * D : 0;
    static constexpr int kBarOff = kStageOff + kStageBytes;
    // kv_full[S] kv_empty[S] q_full q_empty s_full[2] p_full[2] o_full[2] o_empty[2] done uq_full[4] uq_empty[4]
    // v_fixed[kFixRing] vlast_full[kVlast] vlast_empty[kVlast] cp_full epi_done[2]
    static constexpr int kNumBars = 2 * kSlots + 11 + 2 * kUnitQueue + kFixRing + 2 * kVlast + 1 + 2;
    static constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 64 + kUnitQueue * 64 + 1024;
    static constexpr uint32_t kTmemCols = 512;                  // S_A 0, O_A 128, S_B 256, O_B 384
                                                                // (P_X, bf16, overwrites the first 64 columns of S_X)
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// Which pairs of a 32-key chunk take exp2 on the FMA pipe (exp2_poly2) rather than the special-function unit:
// kPolyPairs of the 16, spread evenly.  ex2 on the special-function unit is the scarce resource of the
// softmax (two 128-key rows per thread and key tile, one per Q tile); the polynomial costs about five
// FMA-pipe instructions per element instead.
constexpr int kPolyPairs = 0;
__host__ __device__ constexpr bool poly_pair(int i) { return ((i + 1) * kPolyPairs) / 16 != (i * kPolyPairs) / 16; }

__device__ __forceinline__ uint32_t col_s(int x) { return x ? 256u : 0u; }
__device__ __forceinline__ uint32_t col_o(int x) { return x ? 384u : 128u; }

struct Unit {                 // 16 words; copied through the shared-memory unit queue
    int valid;
    int s, kvh;
    int q0;          // row of the sequence's first new token in q / out
    int n_new, n_k, c;
    int kbeg;        // first key of the unit's key range (a multiple of 128)
    int chunk;       // key chunk index (0 unless the key range is split)
    int tok0[2];     // first new token of tile A / B (relative to the sequence)
    int kend[2];     // keys [kbeg, kend) visible to some row of the tile (kend = kbeg: tile absent)
    int nt[2];       // key tiles of tile A / B
    int nk;          // key tiles loaded for the unit
};
static_assert(sizeof(Unit) == 64, "Unit is copied as 16 words");

__device__ __forceinline__ Unit unit_from_record(const PrefillArgs &a, int4 rec, int4 geo, int TQ) {
    Unit U;
    U.valid = 0;
    U.s = rec.x;
    U.kvh = rec.y;
    const int r = rec.z;
    U.chunk = rec.w;
    if (!geo.w) return U;
    U.q0 = geo.x;
    U.n_new = geo.y;
    U.n_k = geo.z;
    U.c = U.n_k - U.n_new;
    const int npairs = (U.n_new + 2 * TQ - 1) / (2 * TQ);
    if (r >= npairs) return U;
    const int p = npairs - 1 - r;
    // key range: the whole context, or one chunk of it when a non-causal call splits the keys
    U.kbeg = a.key_chunk > 0 ? U.chunk * a.key_chunk : 0;
    const int kmax = a.key_chunk > 0 ? min(U.n_k, U.kbeg + a.key_chunk) : U.n_k;
    for (int x = 0; x < 2; ++x) {
        U.tok0[x] = (2 * p + x) * TQ;
        const int nq = max(0, min(TQ, U.n_new - U.tok0[x]));
        U.kend[x] = nq == 0 ? U.kbeg : (a.causal ? U.c + U.tok0[x] + nq : kmax);
        U.nt[x] = (U.kend[x] - U.kbeg + kN - 1) / kN;
    }
    U.nk = max(U.nt[0], U.nt[1]);
    U.valid = 1;
    return U;
}

// kFused: pa_store_kv_prefill_varlen.  Keys past the cached prefix come from the new K/V rows (tm_kn, tm_vn)
// instead of the cache, and the V-fix warp stores each unit's own new rows to their cache slots.
// kPartial: the key range is cut into chunks and each writes fp32 partials with their log-sum-exp (a.part_o,
// a.part_lse) instead of bf16 rows (the shared-prefix phase of pa_decode_shared_prefix).
template <int D, bool kFused, bool kPartial>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kn,
                   const __grid_constant__ CUtensorMap tm_vn, const PrefillArgs a) {
    using C = PrefillCfg<D, kFused>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *kv_full = bars;
    uint64_t *kv_empty = bars + C::kSlots;
    uint64_t *q_full = bars + 2 * C::kSlots;
    uint64_t *q_empty = q_full + 1;
    uint64_t *s_full = q_empty + 1;    // [2]
    uint64_t *p_full = s_full + 2;     // [2]
    uint64_t *o_full = p_full + 2;     // [2]
    uint64_t *o_empty = o_full + 2;    // [2]
    uint64_t *done = o_empty + 2;
    uint64_t *uq_full = done + 1;      // [kUnitQueue]
    uint64_t *uq_empty = uq_full + kUnitQueue;
    uint64_t *v_fixed = uq_empty + kUnitQueue;   // [kFixRing] the last V tile of a unit is ready for PV
    // The last V tile of a unit lands on its own barrier, from a ring of kVlast taken in unit order: the V-fix
    // warp arrives on the matching vlast_empty once it has waited, and the K/V warp waits for that before it
    // reuses the entry, so every phase is waited for in order whatever the K/V warp's lead.
    uint64_t *vlast_full = v_fixed + kFixRing;    // [kVlast]
    uint64_t *vlast_empty = vlast_full + kVlast;  // [kVlast]
    uint64_t *cp_full = vlast_empty + kVlast;     // fused store: a copy round's rows are in the staging area
    // partial results: softmax warpgroup X has written its tile's partials out of the Q_X buffer (the next unit's
    // Q may be loaded over it)
    uint64_t *epi_done = cp_full + 1;             // [2]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::kNumBars);
    // set by the first wait of this CTA that gives up; every other wait then gives up at once
    volatile int32_t *abort_flag = reinterpret_cast<volatile int32_t *>(tmem_slot + 1);
    // unit queue: kUnitQueue entries of 16 words (a decoded Unit; valid = -1 ends the stream)
    volatile int32_t *unit_q = reinterpret_cast<volatile int32_t *>(tmem_slot + 16);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.group;
    const int TQ = kM / G;
    int32_t *plan_w = static_cast<int32_t *>(a.workspace);
    const PlanLayout plan = plan_layout(a.ranks, a.batch);

    const uint32_t sbase = smem_u32(smem);
    const uint32_t q_s = sbase + C::kQOff;
    const uint32_t ring = sbase + C::kRingOff;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int i = 0; i < C::kSlots; ++i) {
            mbar_init(smem_u32(kv_full + i), 1);
            mbar_init(smem_u32(kv_empty + i), 1);
        }
        mbar_init(smem_u32(q_full), 1);
        mbar_init(smem_u32(q_empty), 1);
        for (int x = 0; x < 2; ++x) {
            mbar_init(smem_u32(s_full + x), 1);
            mbar_init(smem_u32(p_full + x), 4);
            mbar_init(smem_u32(o_full + x), 1);
            mbar_init(smem_u32(o_empty + x), 4);
        }
        mbar_init(smem_u32(done), 1);
        for (int i = 0; i < kFixRing; ++i) mbar_init(smem_u32(v_fixed + i), 1);
        for (int i = 0; i < kVlast; ++i) {
            mbar_init(smem_u32(vlast_full + i), 1);
            mbar_init(smem_u32(vlast_empty + i), 1);
        }
        mbar_init(smem_u32(cp_full), 1);
        for (int x = 0; x < 2; ++x) mbar_init(smem_u32(epi_done + x), 4);
        for (int i = 0; i < kUnitQueue; ++i) {
            mbar_init(smem_u32(uq_full + i), 1);
            mbar_init(smem_u32(uq_empty + i), 11);  // the MMA, V-fix and Q warps, the eight softmax warps
        }
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // everything above overlapped the planning kernel; its table (and all earlier work) is visible after this
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // unit hand-out: the TMA warp fetches unit ids, decodes them once and pushes the decoded units
    // (valid = -1 ends the stream); the other roles pop them in order
    auto pop_unit = [&](uint32_t k, bool arrive, Unit &U) -> bool {
        const int slot = k % kUnitQueue;
        if (!mbar_wait(smem_u32(uq_full + slot), (k / kUnitQueue) & 1, a.dev_error, 0xffffffffu, abort_flag)) return false;
        int32_t *dst = reinterpret_cast<int32_t *>(&U);
#pragma unroll
        for (int i = 0; i < 16; ++i) dst[i] = unit_q[slot * 16 + i];
        __syncwarp();
        if (arrive) mbar_arrive(smem_u32(uq_empty + slot));
        return U.valid >= 0;
    };

    if (warp >= 8) {
        // the third warpgroup (TMA, MMA and V-fix warps, and the spare warp, which has no role) gives
        // registers back to the softmax warpgroups; all four warps run this one instruction
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
        if (warp == kTmaWarp) {
            // ============================================================ TMA ==
            // The whole warp runs this role: every lane waits on the barriers, lane 0 issues the copies, and
            // block ids are read 32 at a time (one per lane) and passed around with shuffles.
            if (lane == 0) {
                tma_prefetch_desc(&tm_q);
                tma_prefetch_desc(&tm_k);
                tma_prefetch_desc(&tm_v);
            }
            const int B = a.block_size, box = a.box_tokens;
            const int total = plan_w[1];
            const int4 *units = reinterpret_cast<const int4 *>(plan_w + plan.units);
            const int4 *geo = reinterpret_cast<const int4 *>(plan_w + plan.geo);
            auto fetch = [&]() -> int {
                int u = 0;
                if (lane == 0) u = (int)atomicAdd(reinterpret_cast<unsigned int *>(plan_w), 1u);
                return __shfl_sync(0xffffffffu, u, 0);
            };
            auto decode = [&](int u) -> Unit {
                Unit V;
                if (u >= total) {
                    V.valid = -1;
                    return V;
                }
                const int4 rec = units[u];
                return unit_from_record(a, rec, geo[rec.x], TQ);
            };
            uint32_t L = 0, nvlast = 0;
            bool ok = true;
            Unit next = decode(fetch());
            for (uint32_t nu = 0;; ++nu) {
                Unit U = next;
                if (!ok) U.valid = -1;
                const int slot = nu % kUnitQueue;
                if (nu >= (uint32_t)kUnitQueue &&
                    !mbar_wait(smem_u32(uq_empty + slot), (nu / kUnitQueue - 1) & 1, a.dev_error, 0xffffffffu, abort_flag))
                    U.valid = -1;
                if (lane == 0) {
                    const int32_t *src = reinterpret_cast<const int32_t *>(&U);
#pragma unroll
                    for (int i = 0; i < 16; ++i) unit_q[slot * 16 + i] = src[i];
                    mbar_arrive(smem_u32(uq_full + slot));
                }
                __syncwarp();
                if (U.valid < 0) break;
                // take the next unit now; its id and record loads overlap this unit's copies
                const int next_u = fetch();
                if (U.valid) {
                    // K and V only (the Q warp loads Q): this warp runs ahead into the next units as far as the
                    // ring slots, the unit queue and the last-V ring let it, so a unit's first tiles are loaded
                    // while the previous unit still computes
                    const int32_t *bt = a.block_table + (int64_t)U.s * a.bt_stride;
                    const int kend = max(U.kend[0], U.kend[1]);
                    int chunk = -32, ids = 0;            // block_table[chunk + lane] lives in `ids` of that lane
                    if (ok && U.nk > 0) ++nvlast;
                    const int nloads = 2 * U.nk;
                    for (int li = 0; li < nloads && ok; ++li) {
                        const int j = li >> 1, kv = li & 1;
                        const int key0 = U.kbeg + j * kN;
                        const int nbox = (min(kN, kend - key0) + box - 1) / box;
                        const int last_blk = (key0 + (nbox - 1) * box) / B;
                        if (last_blk >= chunk + 32) {
                            chunk = key0 / B;
                            ids = chunk + lane < a.bt_stride ? bt[chunk + lane] : -1;
                        }
                        const int slot2 = L % C::kSlots;
                        if (L >= (uint32_t)C::kSlots &&
                            !mbar_wait(smem_u32(kv_empty + slot2), (L / C::kSlots - 1) & 1, a.dev_error, 0xffffffffu, abort_flag)) {
                            ok = false;
                            break;
                        }
                        // the last V tile of the unit lands on its own barrier (the V-fix warp consumes it in
                        // order); the ring slot's barrier still completes one phase, with no bytes
                        const bool vlast = kv == 1 && j == U.nk - 1;
                        if (vlast && nvlast > (uint32_t)kVlast &&
                            !mbar_wait(smem_u32(vlast_empty + (nvlast - 1) % kVlast), ((nvlast - 1) / kVlast - 1) & 1,
                                       a.dev_error, 0xffffffffu, abort_flag)) {
                            ok = false;
                            break;
                        }
                        const uint32_t fb = smem_u32(vlast ? vlast_full + (nvlast - 1) % kVlast : kv_full + slot2);
                        if (lane == 0) {
                            if (vlast) mbar_arrive(smem_u32(kv_full + slot2));
                            mbar_arrive_expect_tx(fb, (uint32_t)(nbox * box * kRowBytes * C::kHalves));
                        }
                        __syncwarp();                        // the expected bytes are posted before any copy
                        const uint32_t dst = ring + slot2 * C::kTileBytes;
                        // one box (block_size tokens, or 128 for larger blocks) per lane: with small blocks a
                        // tile is many boxes, and one issuing thread would fall behind the tensor cores
                        for (int b0 = 0; b0 < nbox; b0 += 32) {
                            const int b = b0 + lane;
                            const int tok = key0 + b * box;
                            const int blk = __shfl_sync(0xffffffffu, ids, b < nbox ? tok / B - chunk : 0);
                            if (b < nbox) {
                                int row;
                                const CUtensorMap *map = kv ? &tm_v : &tm_k;
                                if (kFused && tok >= U.c) {
                                    // a new key: row q0 + (tok - c) of the new K/V (a box never straddles c,
                                    // which is a whole number of blocks); rows past the tensor read zeros
                                    row = U.q0 + (tok - U.c);
                                    map = kv ? &tm_vn : &tm_kn;
                                } else if ((unsigned)blk < (unsigned)a.num_blocks) {
                                    row = blk * B + (tok % B);
                                } else {
                                    report(a.dev_error, PA_DEVERR_BLOCK_ID);
                                    row = -box;     // fully out of range: TMA fills zeros
                                }
#pragma unroll
                                for (int h = 0; h < C::kHalves; ++h)
                                    tma_load_3d(dst + h * kSlab + b * box * kRowBytes, map, h * 64, U.kvh, row, fb);
                            }
                        }
                        ++L;
                    }
                }
                next = decode(next_u);
            }
            // Leave no TMA copy in flight: wait (bounded) for the last load of every ring slot and of every
            // last-V barrier.  On the normal path the MMA and V-fix warps consumed them all and these return at
            // once; they ignore the abort flag, since the copies land in this CTA's shared memory whatever
            // happened.
            for (uint32_t i = (L > (uint32_t)C::kSlots ? L - C::kSlots : 0); i < L; ++i)
                mbar_wait(smem_u32(kv_full + i % C::kSlots), (i / C::kSlots) & 1, a.dev_error);
            for (uint32_t i = (nvlast > (uint32_t)kVlast ? nvlast - kVlast : 0); i < nvlast; ++i)
                mbar_wait(smem_u32(vlast_full + i % kVlast), (i / kVlast) & 1, a.dev_error);
        } else if (warp == kQWarp) {
            // ============================================================== Q ==
            // Both Q tiles of each unit, as soon as the previous unit's S products have read the buffer.
            // With partial results (kPartial) the softmax warpgroups stage their epilogue in the Q buffer, so a
            // unit's Q also waits until the previous unit's tiles have been written out of it.
            if (lane == 0) tma_prefetch_desc(&tm_q);
            uint32_t nq = 0, ne[2] = {0, 0};
            int prev_nt[2] = {0, 0};
            for (uint32_t k = 0;; ++k) {
                Unit U;
                if (!pop_unit(k, lane == 0, U)) break;
                if (!U.valid) continue;
                if (nq > 0 && !mbar_wait(smem_u32(q_empty), (nq - 1) & 1, a.dev_error, 0xffffffffu, abort_flag)) break;
                bool epi_ok = true;
                for (int x = 0; x < 2 && epi_ok; ++x)
                    if (kPartial && prev_nt[x] > 0) {
                        epi_ok = mbar_wait(smem_u32(epi_done + x), ne[x] & 1, a.dev_error, 0xffffffffu, abort_flag);
                        ++ne[x];
                    }
                if (!epi_ok) break;
                prev_nt[0] = U.nt[0];
                prev_nt[1] = U.nt[1];
                if (lane == 0) {
                    mbar_arrive_expect_tx(smem_u32(q_full), (uint32_t)(2 * C::kTileBytes));
                    for (int x = 0; x < 2; ++x)
#pragma unroll
                        for (int h = 0; h < C::kHalves; ++h)
                            tma_load_3d(q_s + x * C::kTileBytes + h * kSlab, &tm_q, h * 64, U.kvh * G, U.q0 + U.tok0[x],
                                        smem_u32(q_full));
                }
                __syncwarp();
                ++nq;
            }
            // the last Q load has landed before the CTA can exit (bounded; ignores the abort flag)
            if (nq > 0) mbar_wait(smem_u32(q_full), (nq - 1) & 1, a.dev_error);
        } else if (warp == kMmaWarp) {
            // ============================================================ MMA ==
            // One thread: the tensor cores keep almost no queue, so this thread does nothing but wait for
            // its operands and issue.  Order per key tile j: PV_A(j) S_A(j+1) PV_B(j) S_B(j+1).
            if (lane == 0) {
                constexpr uint32_t idesc_qk = idesc_bf16_f32(kM, kN, 0, 0);
                constexpr uint32_t idesc_pv = idesc_bf16_f32(kM, D, 0, 1);
                uint32_t nq = 0, L = 0, np[2] = {0, 0}, no[2] = {0, 0}, nfix = 0;
                bool ok = true;
                // Descriptors are built once; an MMA only adds a byte offset (>> 4) to the start-address
                // field (14 bits of a 256 KB window, so the add never carries into the other fields).
                const uint64_t q_desc = smem_desc_sw128(q_s, 16, 1024);
                const uint64_t k_desc = smem_desc_sw128(ring, 16, 1024);
                const uint64_t v_desc = smem_desc_sw128(ring, kSlab, 1024);
                auto wait_slot = [&](uint32_t idx) -> bool {
                    return mbar_wait(smem_u32(kv_full + idx % C::kSlots), (idx / C::kSlots) & 1, a.dev_error, 0xffffffffu, abort_flag);
                };
                auto issue_s = [&](int x, uint32_t kidx) {
                    const uint64_t qd = q_desc + ((uint32_t)(x * C::kTileBytes) >> 4);
                    const uint64_t kd = k_desc + (((kidx % C::kSlots) * (uint32_t)C::kTileBytes) >> 4);
                    const uint32_t d = tmem + col_s(x);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = ((kk >> 2) * kSlab + (kk & 3) * 32) >> 4;
                        tc_mma_ss(d, qd + off, kd + off, idesc_qk, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(smem_u32(s_full + x));
                };
                auto issue_pv = [&](int x, uint32_t vidx, bool accumulate) {
                    const uint64_t vd = v_desc + (((vidx % C::kSlots) * (uint32_t)C::kTileBytes) >> 4);
                    const uint32_t d = tmem + col_o(x), pa = tmem + col_s(x);
#pragma unroll
                    for (int kk = 0; kk < kN / 16; ++kk) {
                        // A = P_X in TMEM: 16 keys = 8 columns of packed bf16 pairs; B = V rows kk*16 ..
                        tc_mma_ts(d, pa + kk * 8, vd + ((kk * 16 * kRowBytes) >> 4), idesc_pv,
                                  (accumulate || kk > 0) ? 1u : 0u);
                    }
                };
                for (uint32_t k = 0; ok; ++k) {
                    const int slot = k % kUnitQueue;
                    if (!mbar_wait(smem_u32(uq_full + slot), (k / kUnitQueue) & 1, a.dev_error, 0xffffffffu, abort_flag)) break;
                    Unit U;
                    {
                        int32_t *dst = reinterpret_cast<int32_t *>(&U);
#pragma unroll
                        for (int i = 0; i < 16; ++i) dst[i] = unit_q[slot * 16 + i];
                    }
                    mbar_arrive(smem_u32(uq_empty + slot));
                    if (U.valid < 0) break;
                    if (!U.valid) continue;
                    if (!mbar_wait(smem_u32(q_full), nq & 1, a.dev_error, 0xffffffffu, abort_flag)) break;
                    ++nq;
                    const bool hasB = U.nt[1] > 0;
                    // K_0: S_A(0), S_B(0)
                    if (!wait_slot(L)) break;
                    tc_fence_after();
                    issue_s(0, L);
                    if (hasB) issue_s(1, L);
                    tc_commit(smem_u32(kv_empty + L % C::kSlots));
                    if (U.nk == 1) tc_commit(smem_u32(q_empty));
                    for (int j = 0; j < U.nk && ok; ++j) {
                        const uint32_t vidx = L + 2 * j + 1, knext = L + 2 * j + 2;
                        if (j == U.nk - 1) {
                            // the V-fix warp has zeroed the rows past the key range of the unit's last V tile
                            if (!mbar_wait(smem_u32(v_fixed + nfix % kFixRing), (nfix / kFixRing) & 1, a.dev_error,
                                           0xffffffffu, abort_flag)) {
                                ok = false;
                                break;
                            }
                            ++nfix;
                        } else if (!wait_slot(vidx)) {
                            ok = false;
                            break;
                        }
                        bool knext_ready = false;
                        for (int x = 0; x < 2; ++x) {
                            if (j >= U.nt[x]) continue;
                            if (!mbar_wait(smem_u32(p_full + x), np[x] & 1, a.dev_error, 0xffffffffu, abort_flag)) { ok = false; break; }
                            ++np[x];
                            if (j == 0 && no[x] > 0 &&
                                !mbar_wait(smem_u32(o_empty + x), (no[x] - 1) & 1, a.dev_error, 0xffffffffu, abort_flag)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            issue_pv(x, vidx, j > 0);
                            if (j == U.nt[x] - 1) {
                                tc_commit(smem_u32(o_full + x));
                                ++no[x];
                            }
                            if (j + 1 < U.nt[x]) {
                                if (!knext_ready) {
                                    if (!wait_slot(knext)) { ok = false; break; }
                                    tc_fence_after();
                                    knext_ready = true;
                                }
                                issue_s(x, knext);
                            }
                        }
                        if (!ok) break;
                        tc_commit(smem_u32(kv_empty + vidx % C::kSlots));
                        if (knext_ready) tc_commit(smem_u32(kv_empty + knext % C::kSlots));
                        if (j == U.nk - 2) tc_commit(smem_u32(q_empty));   // every S product of the unit is issued
                    }
                    L += 2 * U.nk;
                }
                // every MMA issued by this thread has completed before TMEM is freed
                tc_commit(smem_u32(done));
                mbar_wait(smem_u32(done), 0, a.dev_error);
            }
        } else if (warp == kFixWarp) {
            // ========================================================== V fix ==
            // Zero the rows of each unit's last V tile past its key range (stale or poisoned cache slots),
            // so that masked keys, whose probabilities are exactly 0, never meet a NaN.
            // Fused store: between those fixes this warp copies each unit's own new tokens' K/V rows of its KV
            // head to their cache slots with the bulk-copy engine, in rounds of up to kStageTokens tokens:
            // bulk loads of the rows into the staging area (completing on cp_full), then one bulk store per
            // row to its slot.  The warp never waits on a copy while a fix is due -- it polls for the next
            // unit's last V tile between steps -- so the MMA waits for fixes only.  Units whose rows are not
            // yet copied wait in a small FIFO; the rest is copied when the CTA has no unit left.  No kernel of
            // this launch reads those slots.
            uint32_t L = 0, nfx = 0;
            constexpr int kFifo = 4;
            int fq_s[kFifo], fq_kvh[kFifo], fq_q0[kFifo], fq_c[kFifo], fq_i[kFifo], fq_end[kFifo];
            int fq_head = 0, fq_n = 0;            // oldest entry, entries in use
            int cp_state = 0;                     // 0: staging free, 1: loads in flight, 2: stores issued
            uint32_t cp_rounds = 0;               // completed phases of cp_full
            int rd_s = 0, rd_kvh = 0, rd_q0 = 0, rd_c = 0, rd_i = 0, rd_n = 0;   // the round in flight
            const uint32_t stage = sbase + C::kStageOff;
            const uint32_t cpb = smem_u32(cp_full);
            // take up to kStageTokens tokens of the oldest pending unit and start their loads
            auto start_round = [&]() {
                int end = 0;
#pragma unroll
                for (int e = 0; e < kFifo; ++e)
                    if (e == fq_head) {
                        rd_s = fq_s[e];
                        rd_kvh = fq_kvh[e];
                        rd_q0 = fq_q0[e];
                        rd_c = fq_c[e];
                        rd_i = fq_i[e];
                        end = fq_end[e];
                    }
                rd_n = min(C::kStageTokens, end - rd_i);
#pragma unroll
                for (int e = 0; e < kFifo; ++e)
                    if (e == fq_head) fq_i[e] = rd_i + rd_n;
                if (rd_i + rd_n >= end) {
                    fq_head = (fq_head + 1) % kFifo;
                    --fq_n;
                }
                if (lane == 0) mbar_arrive_expect_tx(cpb, (uint32_t)(rd_n * 4 * D));
                __syncwarp();
                for (int t = lane; t < rd_n; t += 32) {
                    const int64_t row = (int64_t)rd_q0 + rd_i + t;
                    bulk_load(stage + t * 4 * D,
                              static_cast<const __nv_bfloat16 *>(a.k_new) + row * a.kn_stride + (int64_t)rd_kvh * D, 2 * D,
                              cpb);
                    bulk_load(stage + t * 4 * D + 2 * D,
                              static_cast<const __nv_bfloat16 *>(a.v_new) + row * a.vn_stride + (int64_t)rd_kvh * D, 2 * D,
                              cpb);
                }
                cp_state = 1;
            };
            // the round's rows have landed: one bulk store per row to its slot
            auto store_round = [&]() {
                mbar_wait(cpb, cp_rounds & 1, a.dev_error);   // returns at once: every lane acquires the rows
                ++cp_rounds;
                for (int t = lane; t < rd_n; t += 32) {
                    const int64_t row = (int64_t)rd_q0 + rd_i + t;
                    const int32_t sl = __ldg(a.new_slots + row);
                    if (sl < 0 || (int64_t)sl >= a.num_slots) {
                        report(a.dev_error, PA_DEVERR_SLOT);   // not stored
                        continue;
                    }
                    if (a.dev_error) {   // the slot must be the row this prefill read as key c + i
                        const int pos = rd_c + rd_i + t;
                        const int32_t blk = __ldg(a.block_table + (int64_t)rd_s * a.bt_stride + pos / a.block_size);
                        if ((int64_t)sl != (int64_t)blk * a.block_size + pos % a.block_size) report(a.dev_error, PA_DEVERR_SLOT);
                    }
                    const int64_t off = ((int64_t)sl * a.num_kv_heads + rd_kvh) * D;
                    bulk_store(static_cast<__nv_bfloat16 *>(a.k_cache) + off, stage + t * 4 * D, 2 * D);
                    bulk_store(static_cast<__nv_bfloat16 *>(a.v_cache) + off, stage + t * 4 * D + 2 * D, 2 * D);
                }
                bulk_commit();
                cp_state = 2;
            };
            // One loop, one site for each copy step.  With no unit left it drains the FIFO.
            bool more = true;
            for (uint32_t k = 0;; ++k) {
                Unit U;
                U.valid = 0;
                if (more && !pop_unit(k, lane == 0, U)) more = false;
                if (more && !U.valid) continue;
                const uint32_t vbar = smem_u32(vlast_full + nfx % kVlast), vpar = (nfx / kVlast) & 1;
                if (kFused) {
                    // pump the copy engine until the unit's last V tile lands (a fix first, always) or, with
                    // no unit left, until nothing is pending; leave room in the FIFO for this unit.  Bounded:
                    // polls sleep 128 ns and a round's loads are waited for at most kWaitTimeoutNs.
                    uint64_t t_loads = 0;
                    for (;;) {
                        if (more && fq_n < kFifo && __any_sync(0xffffffffu, mbar_test_wait(vbar, vpar))) break;
                        if (cp_state == 1) {
                            const bool landed = __any_sync(0xffffffffu, mbar_test_wait(cpb, cp_rounds & 1));
                            if (landed || !more || (t_loads && global_timer_ns() - t_loads > kWaitTimeoutNs)) {
                                store_round();
                                t_loads = 0;
                            } else {
                                if (!t_loads) t_loads = global_timer_ns();
                                __nanosleep(128);
                            }
                            continue;
                        }
                        if (cp_state == 2) {          // the staging area is free once the stores have read it
                            bulk_wait_read();
                            __syncwarp();
                            cp_state = 0;
                            continue;
                        }
                        if (fq_n > 0) {
                            start_round();
                            continue;
                        }
                        break;                        // nothing pending
                    }
                }
                if (!more) break;
                const uint32_t vidx = L + 2 * (U.nk - 1) + 1;
                L += 2 * U.nk;
                if (!mbar_wait(vbar, vpar, a.dev_error, 0xffffffffu, abort_flag)) break;
                if (lane == 0) mbar_arrive(smem_u32(vlast_empty + nfx % kVlast));   // the entry may be reused
                ++nfx;
                const int valid = max(U.kend[0], U.kend[1]) - (U.kbeg + (U.nk - 1) * kN);
                if (valid < kN) {
                    const uint32_t vs = ring + (vidx % C::kSlots) * C::kTileBytes;
                    for (int e = lane; e < (kN - valid) * C::kHalves * 8; e += 32) {
                        const int r = valid + e / (C::kHalves * 8);
                        const int h = (e / 8) % C::kHalves, ch = e % 8;
                        asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(vs + h * kSlab + r * kRowBytes + ch * 16),
                                     "r"(0u)
                                     : "memory");
                    }
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(v_fixed + (nfx - 1) % kFixRing));
                if (kFused && U.chunk == 0) {
                    // this unit's own tokens: tile A's, then tile B's (present only when tile A is full); the
                    // loop above left room in the FIFO
                    const int e_new = (fq_head + fq_n) % kFifo;
                    const int i0 = U.tok0[0], i1 = min(U.n_new, U.tok0[0] + 2 * TQ);
#pragma unroll
                    for (int e = 0; e < kFifo; ++e)
                        if (e == e_new) {
                            fq_s[e] = U.s;
                            fq_kvh[e] = U.kvh;
                            fq_q0[e] = U.q0;
                            fq_c[e] = U.c;
                            fq_i[e] = i0;
                            fq_end[e] = i1;
                        }
                    if (i1 > i0) ++fq_n;
                }
            }
            if (kFused) {
                // leave nothing in flight: the last round's loads (bounded), then every bulk store
                if (cp_state == 1) mbar_wait(cpb, cp_rounds & 1, a.dev_error);
                bulk_wait_all();
            }
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
        // ======================================================== softmax ==
        const int x = warp >> 2;                       // 0: tile A, 1: tile B
        const int r = threadIdx.x & 127;               // TMEM lane == Q-tile row
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const float sl = a.scale_log2;
        uint32_t ns = 0, no = 0;
        for (uint32_t k = 0;; ++k) {
            Unit U;
            if (!pop_unit(k, lane == 0, U)) break;
            if (!U.valid || U.nt[x] == 0) continue;
            const int t = U.tok0[x] + r / G;              // this row's new-token index
            int lim = a.causal ? U.c + t : U.n_k - 1;      // last visible key
            if (lim > U.kend[x] - 1) lim = U.kend[x] - 1;  // never past the unit's key range
            float m_ref = -INFINITY, l = 0.f;
            bool ok = true;
            for (int j = 0; j < U.nt[x]; ++j) {
                if (!mbar_wait(smem_u32(s_full + x), ns & 1, a.dev_error, 0xffffffffu, abort_flag)) { ok = false; break; }
                ++ns;
                tc_fence_after();
                uint32_t sr[4][32];   // the S row: one 128-column TMEM load (measured ~2 % faster than four)
                tmem_ld128(lane_base + col_s(x), reinterpret_cast<uint32_t (&)[128]>(sr));
                tc_wait_ld();
                const int thr = lim - (U.kbeg + j * kN);   // keys e <= thr are visible
                // row maximum: three-input max over pairs, four independent chains
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                if (thr >= kN - 1) {
#pragma unroll
                    for (int e = 0; e < kN; e += 8)
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            mx[c] = max3f(mx[c], __uint_as_float(sr[(e + 2 * c) >> 5][(e + 2 * c) & 31]),
                                          __uint_as_float(sr[(e + 2 * c + 1) >> 5][(e + 2 * c + 1) & 31]));
                } else {
#pragma unroll
                    for (int e = 0; e < kN; ++e) {
                        const float v = e <= thr ? __uint_as_float(sr[e >> 5][e & 31]) : -INFINITY;
                        sr[e >> 5][e & 31] = __float_as_uint(v);
                        mx[e & 3] = fmaxf(mx[e & 3], v);
                    }
                }
                const float m_new = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl;
                float corr = 1.f;
                bool rescale = false;
                if (m_new > m_ref + 8.f) {                  // also true while m_ref is -inf
                    corr = fast_exp2(m_ref - m_new);
                    m_ref = m_new;
                    rescale = true;
                }
                // P = exp2(s * scale_log2 - m_ref) as packed bf16 pairs, written over the S_X columns already
                // read (64 keys = 32 columns per store); the scaling runs on pairs (f32x2 FMA).  The row sum
                // adds the bf16 values the PV product multiplies, not the fp32 ones, so that the weights of the
                // numerator and the denominator are the same numbers: with the lazy maximum the largest P is not
                // a power of two, and its rounding would otherwise show in the output of a row that one key
                // dominates.
                const uint64_t sl2 = f2_pack(sl, sl), neg2 = f2_pack(-m_ref, -m_ref);
                uint64_t ls2[2] = {0ull, 0ull};
                uint32_t w2[32];   // P of 64 keys (32 columns), stored with one instruction per pair of chunks
#pragma unroll
                for (int kc = 0; kc < kN / 32; ++kc) {
                    uint32_t *w = w2 + (kc & 1) * 16;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const uint64_t x2 =
                            f2_fma(f2_pack(__uint_as_float(sr[kc][2 * i]), __uint_as_float(sr[kc][2 * i + 1])), sl2, neg2);
                        float p0, p1;
                        if (poly_pair(i)) {
                            f2_unpack(exp2_poly2(x2), p0, p1);
                        } else {
                            f2_unpack(x2, p0, p1);
                            p0 = fast_exp2(p0);
                            p1 = fast_exp2(p1);
                        }
                        w[i] = pack_bf16(p0, p1);
                        ls2[i & 1] = f2_add(ls2[i & 1], f2_pack(__uint_as_float(w[i] << 16),
                                                                __uint_as_float(w[i] & 0xffff0000u)));
                    }
                    if (kc & 1) tmem_st32(lane_base + col_s(x) + (kc - 1) * 16, w2);
                }
                float ls[4];
                f2_unpack(ls2[0], ls[0], ls[1]);
                f2_unpack(ls2[1], ls[2], ls[3]);
                l = l * corr + ((ls[0] + ls[1]) + (ls[2] + ls[3]));
                // The decision is per row, but tcgen05.ld / st are warp-wide (.sync.aligned): the whole warp
                // takes the branch when any of its rows rescales, and the other rows multiply by corr = 1.
                if (__any_sync(0xffffffffu, rescale && j > 0)) {
                    // O_X is stable: PV_X(j-1) completed before S_X(j), which was issued after it
#pragma unroll
                    for (int q = 0; q < D / 32; ++q) {
                        uint32_t o[32];
                        tmem_ld32(lane_base + col_o(x) + q * 32, o);
                        tc_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
                        tmem_st32(lane_base + col_o(x) + q * 32, o);
                    }
                    tc_wait_st();
                }
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(p_full + x));
            }
            if (!ok) break;
            // ---- epilogue: O / l -> bf16 rows ----
            if (!mbar_wait(smem_u32(o_full + x), no & 1, a.dev_error, 0xffffffffu, abort_flag)) break;
            ++no;
            tc_fence_after();
            const float inv = 1.f / l;
            const bool store = t < U.n_new;
            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out) +
                                                   ((int64_t)(U.q0 + (store ? t : 0)) * a.num_q_heads +
                                                    (int64_t)U.kvh * G + r % G) * D);
            if (kPartial) {
                // partial result of this key chunk: fp32 O / l and its log-sum-exp (log2 units), to be merged
                // with the other partials of the same (query, head).  A thread holds one 512-byte row; written
                // straight out, every warp store would touch 32 rows.  So the warp stages 32 columns of its 32
                // rows at a time in its 4 KB of the Q_X buffer (free: every S product of this unit has completed
                // before o_full; the Q warp waits for epi_done before loading over it), 16-byte pieces swizzled
                // by row so that neither side conflicts on banks, and reads them back four rows per instruction:
                // each store instruction then writes four whole 128-byte lines.
                const int64_t pi = store ? ((int64_t)(U.q0 + t) * a.num_q_heads + (int64_t)U.kvh * G + r % G) *
                                               a.part_slots + a.part_base + U.chunk
                                         : 0;
                const uint32_t smask = __ballot_sync(0xffffffffu, store);
                const uint32_t stg = q_s + (uint32_t)(x * C::kTileBytes) + (uint32_t)((warp & 3) * 4096);
                const int c = lane & 7;
#pragma unroll 1
                for (int q = 0; q < D / 32; ++q) {
                    uint32_t oq[32];   // 32 columns of O_X at a time (units per CTA are few here: O_X is released after)
                    tmem_ld32(lane_base + col_o(x) + q * 32, oq);
                    tc_wait_ld();
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(stg + lane * 128 + ((e ^ (lane & 7)) << 4)),
                                     "f"(__uint_as_float(oq[4 * e]) * inv), "f"(__uint_as_float(oq[4 * e + 1]) * inv),
                                     "f"(__uint_as_float(oq[4 * e + 2]) * inv), "f"(__uint_as_float(oq[4 * e + 3]) * inv)
                                     : "memory");
                    __syncwarp();
#pragma unroll 4
                    for (int i = 0; i < 8; ++i) {
                        const int rr = i * 4 + (lane >> 3);          // the warp's row this lane writes 16 bytes of
                        const int64_t pr = __shfl_sync(0xffffffffu, pi, rr);
                        float4 v;
                        asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                     : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                                     : "r"(stg + rr * 128 + ((c ^ (rr & 7)) << 4))
                                     : "memory");
                        if ((smask >> rr) & 1) reinterpret_cast<float4 *>(a.part_o + pr * D + q * 32)[c] = v;
                    }
                    __syncwarp();
                }
                tc_fence_before();
                if (store) a.part_lse[pi] = m_ref + __log2f(l);
                fence_proxy_async_smem();   // the next Q copy (async proxy) lands where this warp wrote
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(smem_u32(o_empty + x));
                    mbar_arrive(smem_u32(epi_done + x));
                }
            } else {
                uint32_t o[D / 32][32];
#pragma unroll
                for (int q = 0; q < D / 32; ++q) tmem_ld32(lane_base + col_o(x) + q * 32, o[q]);
                tc_wait_ld();
                // O_X is in registers: hand its TMEM columns back to the MMA thread now, so that the next unit's
                // first PV product does not wait for the global stores below
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(o_empty + x));
                if (store) {
#pragma unroll
                    for (int q = 0; q < D / 32; ++q)
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            uint4 v;
                            v.x = pack_bf16(__uint_as_float(o[q][e]) * inv, __uint_as_float(o[q][e + 1]) * inv);
                            v.y = pack_bf16(__uint_as_float(o[q][e + 2]) * inv, __uint_as_float(o[q][e + 3]) * inv);
                            v.z = pack_bf16(__uint_as_float(o[q][e + 4]) * inv, __uint_as_float(o[q][e + 5]) * inv);
                            v.w = pack_bf16(__uint_as_float(o[q][e + 6]) * inv, __uint_as_float(o[q][e + 7]) * inv);
                            dst[(q * 32 + e) / 8] = v;
                        }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}


template <int D>
cudaError_t launch_prefill_d(const PrefillArgs &a, const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                             const CUtensorMap &tm_v, const CUtensorMap &tm_kn, const CUtensorMap &tm_vn,
                             cudaStream_t stream) {
    const bool fused = a.new_slots != nullptr;
    const int mode = fused ? 1 : a.part_o ? 2 : 0;
    auto kernel = mode == 1 ? prefill_kernel<D, true, false> : mode == 2 ? prefill_kernel<D, false, true>
                                                                          : prefill_kernel<D, false, false>;
    const int smem_bytes = fused ? PrefillCfg<D, true>::kSmemBytes : PrefillCfg<D, false>::kSmemBytes;
    static std::atomic<uint64_t> configured[3] = {{0}, {0}, {0}};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = uint64_t(1) << (dev & 63);
    if (!(configured[mode].load(std::memory_order_acquire) & bit)) {
        // the register split inside the kernel assumes the launch-time count it was written for
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, kernel);
        if (e != cudaSuccess) return e;
        if ((uint32_t)fa.numRegs * kThreads < 2 * 128 * kRegsSoftmax + 128 * kRegsOther) return cudaErrorNotSupported;
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
        if (e != cudaSuccess) return e;
        configured[mode].fetch_or(bit, std::memory_order_acq_rel);
    }
    const int TQ = kM / a.group;
    const size_t plan_smem = (size_t)2 * a.batch * sizeof(int32_t);
    prefill_plan_kernel<<<1, kPlanThreads, plan_smem, stream>>>(a, a.ranks, 2 * TQ);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t max_units = (int64_t)a.ranks * a.batch * a.num_kv_heads * a.nchunks;
    const int grid = (int)(max_units < num_sms() ? max_units : num_sms());
    if (grid <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, tm_q, tm_k, tm_v, tm_kn, tm_vn, a);
}

}  // namespace

size_t prefill_workspace_bytes(int32_t batch, int32_t max_seqlen_q, int32_t group, int32_t num_kv_heads,
                               int32_t nchunks) {
    const int32_t TQ = kM / group;
    const int64_t R = ((int64_t)max_seqlen_q + 2 * TQ - 1) / (2 * TQ);
    const PlanLayout lay = plan_layout((int32_t)R, batch);
    const size_t words = (size_t)lay.units + (size_t)4 * R * batch * num_kv_heads * nchunks;
    return (words * sizeof(int32_t) + 255) / 256 * 256;
}

cudaError_t launch_prefill(const PrefillArgs &a, const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                           const CUtensorMap &tm_v, cudaStream_t stream, const CUtensorMap *tm_kn,
                           const CUtensorMap *tm_vn) {
    if (a.new_slots && (!tm_kn || !tm_vn)) return cudaErrorInvalidValue;
    const CUtensorMap &kn = tm_kn ? *tm_kn : tm_k, &vn = tm_vn ? *tm_vn : tm_v;   // unused unless fused
    if (a.head_dim == 128) return launch_prefill_d<128>(a, tm_q, tm_k, tm_v, kn, vn, stream);
    return launch_prefill_d<64>(a, tm_q, tm_k, tm_v, kn, vn, stream);
}

}  // namespace pa
