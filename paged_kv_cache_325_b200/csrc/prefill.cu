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
// How (one CTA per 128-row Q tile):
//  * the 128 MMA rows are (128 / G) consecutive new tokens x the G q-heads
//    of one KV head (GQA packing), so one K/V tile feeds all G heads;
//  * warp 4 (TMA): K/V tiles of 128 keys, gathered block by block through
//    block_table with 3-D tensor-map loads (128-byte swizzle), into a ring
//    of shared-memory stages guarded by mbarriers;
//  * warp 5 (MMA): one thread issues tcgen05.mma.cta_group::1.kind::f16:
//    S = Q K^T (M=128, N=128, K=head_dim) into one of two TMEM S buffers,
//    then O += P V (M=128, N=head_dim, K=128) into the TMEM O accumulator;
//    tcgen05.commit signals the mbarriers;
//  * warps 0-3 (softmax): thread t owns TMEM lane t, i.e. one Q row; it
//    reads its S row with tcgen05.ld, selects masked keys out (-inf), keeps a
//    running max in log2 units and rescales O (tcgen05.ld/st) only when the
//    max grew by more than 8 (2^8), writes P as bf16 into a swizzled
//    shared-memory tile (the A operand of the PV product), and at the end
//    divides O by the row sum and stores bf16 rows to global memory;
//  * V rows of the last key tile beyond the key range are zeroed in shared
//    memory before the PV product, so stale or poisoned cache contents never
//    meet a zero weight (0 * NaN is never formed).
#include <atomic>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr int kM = 128;              // MMA rows per CTA
constexpr int kN = 128;              // keys per K/V tile
constexpr int kThreads = 192;        // 4 softmax warps + TMA warp + MMA warp
constexpr int kTmaWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kRowBytes = 128;       // one 64-element bf16 swizzle row
constexpr int kSlab = kM * kRowBytes;  // 128 rows x 128 B = 16 KB (a 64-column slice of a 128-row tile)

template <int D>
struct PrefillCfg {
    static constexpr int kHalves = D / 64;
    static constexpr int kStages = D == 128 ? 2 : 3;
    static constexpr int kQBytes = kHalves * kSlab;
    static constexpr int kKvBytes = kHalves * kSlab;          // one K (or V) tile of 128 keys
    static constexpr int kStageBytes = 2 * kKvBytes;
    static constexpr int kPBytes = 2 * kSlab;                 // P: 128 rows x 128 keys bf16
    static constexpr int kQOff = 0;
    static constexpr int kRingOff = kQOff + kQBytes;
    static constexpr int kPOff = kRingOff + kStages * kStageBytes;
    static constexpr int kBarOff = kPOff + kPBytes;
    // barriers: kv_full[S], kv_empty[S], s_full[2], s_free[2], p_full, pv_done, + tmem address slot
    static constexpr int kNumBars = 2 * kStages + 6;
    static constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16 + 1024;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const PrefillArgs a) {
    using C = PrefillCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *kv_full = bars;
    uint64_t *kv_empty = bars + C::kStages;
    uint64_t *s_full = bars + 2 * C::kStages;
    uint64_t *s_free = s_full + 2;
    uint64_t *p_full = s_free + 2;
    uint64_t *pv_done = p_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::kNumBars);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.group;
    const int TQ = kM / G;                        // tokens per Q tile
    const int kvh = blockIdx.x % a.num_kv_heads;
    const int s = blockIdx.x / a.num_kv_heads;

    // ---- sequence geometry (validated; a bad sequence is skipped) ----
    const int q0 = __ldg(a.cu_q + s), q1 = __ldg(a.cu_q + s + 1);
    const int k0 = __ldg(a.cu_k + s), k1 = __ldg(a.cu_k + s + 1);
    const int n_new = q1 - q0, n_k = k1 - k0, c = n_k - n_new;
    if (n_new < 0 || c < 0 || q0 < 0 || k0 < 0 || n_new > a.max_seqlen_q || n_k > a.max_seqlen_k ||
        (int64_t)n_k > (int64_t)a.bt_stride * a.block_size) {
        if (blockIdx.y == 0 && kvh == 0 && threadIdx.x == 0) report(a.dev_error, PA_DEVERR_SEQLENS);
        return;
    }
    const int nqt = (n_new + TQ - 1) / TQ;
    if ((int)blockIdx.y >= nqt) return;
    const int qt = nqt - 1 - (int)blockIdx.y;    // blockIdx.y = 0 takes the last (longest) tile
    const int tok0 = qt * TQ;                    // first new token of this tile
    const int nq = min(TQ, n_new - tok0);
    const int kend = a.causal ? c + tok0 + nq : n_k;   // keys [0, kend) are visible to some row
    const int nkt = (kend + kN - 1) / kN;

    const uint32_t sbase = smem_u32(smem);
    const uint32_t q_s = sbase + C::kQOff;
    const uint32_t ring = sbase + C::kRingOff;
    const uint32_t p_s = sbase + C::kPOff;

    // ---- barriers and TMEM ----
    if (threadIdx.x == 0) {
        for (int st = 0; st < C::kStages; ++st) {
            mbar_init(smem_u32(kv_full + st), 1);
            mbar_init(smem_u32(kv_empty + st), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(s_full + b), 1);
            mbar_init(smem_u32(s_free + b), 4);
        }
        mbar_init(smem_u32(p_full), 4);
        mbar_init(smem_u32(pv_done), 1);
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
        tmem_relinquish();
    }

    // ---- Q tile -> shared memory (K-major, 128-byte swizzle), zero rows past n_new ----
    {
        const uint16_t *qg = static_cast<const uint16_t *>(a.q);
        constexpr int kChunksPerRow = D / 8;
        for (int e = threadIdx.x; e < kM * kChunksPerRow; e += kThreads) {
            const int r = e / kChunksPerRow, ch = e % kChunksPerRow;
            const int t = tok0 + r / G;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (t < n_new) {
                const int64_t row = ((int64_t)(q0 + t) * a.num_q_heads + (int64_t)kvh * G + r % G) * D;
                v = __ldg(reinterpret_cast<const uint4 *>(qg + row) + ch);
            }
            const uint32_t dst = q_s + (ch >> 3) * kSlab + swz128(r, ch & 7);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v.x), "r"(v.y), "r"(v.z),
                         "r"(v.w)
                         : "memory");
        }
        fence_proxy_async_smem();   // make the generic-proxy writes visible to the tensor cores
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kTmaWarp) {
        // ============================================================ TMA ==
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            const int32_t *bt = a.block_table + (int64_t)s * a.bt_stride;
            const int B = a.block_size, box = a.box_tokens;
            for (int j = 0; j < nkt; ++j) {
                const int st = j % C::kStages;
                if (j >= C::kStages &&
                    !mbar_wait(smem_u32(kv_empty + st), ((j / C::kStages) & 1) ^ 1, a.dev_error))
                    break;
                const int key0 = j * kN;
                const int nbox = (min(kN, kend - key0) + box - 1) / box;
                const uint32_t fb = smem_u32(kv_full + st);
                mbar_arrive_expect_tx(fb, (uint32_t)(nbox * box * kRowBytes * C::kHalves * 2));
                const uint32_t kd = ring + st * C::kStageBytes, vd = kd + C::kKvBytes;
                for (int b = 0; b < nbox; ++b) {
                    const int tok = key0 + b * box;
                    const int blk = __ldg(bt + tok / B);
                    int row;
                    if ((unsigned)blk < (unsigned)a.num_blocks) {
                        row = blk * B + (tok % B);
                    } else {
                        report(a.dev_error, PA_DEVERR_BLOCK_ID);
                        row = -box;          // fully out of range: TMA fills zeros
                    }
#pragma unroll
                    for (int h = 0; h < C::kHalves; ++h) {
                        const uint32_t off = h * kSlab + b * box * kRowBytes;
                        tma_load_3d(kd + off, &tm_k, h * 64, kvh, row, fb);
                        tma_load_3d(vd + off, &tm_v, h * 64, kvh, row, fb);
                    }
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ============================================================ MMA ==
        constexpr uint32_t idesc_qk = idesc_bf16_f32(kM, kN, 0, 0);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(kM, D, 0, 1);
        bool ok = true;
        auto issue_pv = [&](int jj) -> bool {
            const int st = jj % C::kStages;
            if (!mbar_wait(smem_u32(p_full), jj & 1, a.dev_error)) return false;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t vs = ring + st * C::kStageBytes + C::kKvBytes;
#pragma unroll
                for (int kk = 0; kk < kN / 16; ++kk) {
                    // A = P rows, K-major: key half kk/4, 32-byte step inside the swizzle row
                    const uint64_t ad = smem_desc_sw128(p_s + (kk >> 2) * kSlab + (kk & 3) * 32, 16, 1024);
                    // B = V, MN-major: 16 keys = 2 groups of 8 rows; the D halves are kSlab apart
                    const uint64_t bd = smem_desc_sw128(vs + kk * 16 * kRowBytes, kSlab, 1024);
                    tc_mma_ss(tmem + C::kColO, ad, bd, idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(smem_u32(kv_empty + st));
                tc_commit(smem_u32(pv_done));
            }
            __syncwarp();
            return true;
        };
        for (int j = 0; j < nkt && ok; ++j) {
            const int st = j % C::kStages, b = j & 1;
            if (!mbar_wait(smem_u32(kv_full + st), (j / C::kStages) & 1, a.dev_error)) { ok = false; break; }
            if (j >= 2 && !mbar_wait(smem_u32(s_free + b), ((j >> 1) - 1) & 1, a.dev_error)) { ok = false; break; }
            // last tile: zero the V rows past the key range (stale or poisoned slots)
            const int valid = kend - j * kN;
            if (valid < kN) {
                const uint32_t vs = ring + st * C::kStageBytes + C::kKvBytes;
                for (int e = lane; e < (kN - valid) * C::kHalves * 8; e += 32) {
                    const int r = valid + e / (C::kHalves * 8);
                    const int h = (e / 8) % C::kHalves, ch = e % 8;
                    asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(vs + h * kSlab + r * kRowBytes +
                                                                                   ch * 16),
                                 "r"(0u)
                                 : "memory");
                }
                fence_proxy_async_smem();
                __syncwarp();
            }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t ks = ring + st * C::kStageBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t ad = smem_desc_sw128(q_s + (kk >> 2) * kSlab + (kk & 3) * 32, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(ks + (kk >> 2) * kSlab + (kk & 3) * 32, 16, 1024);
                    tc_mma_ss(tmem + (b ? C::kColS1 : C::kColS0), ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
                }
                tc_commit(smem_u32(s_full + b));
            }
            __syncwarp();
            if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
        }
        if (ok && nkt > 0) issue_pv(nkt - 1);
    } else {
        // ======================================================== softmax ==
        const int r = threadIdx.x;                      // TMEM lane == Q-tile row
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        const int t = tok0 + r / G;                     // this row's new-token index
        int lim = a.causal ? c + t : n_k - 1;           // last visible key
        if (lim > n_k - 1) lim = n_k - 1;               // rows past n_new never see past the keys
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nkt; ++j) {
            const int b = j & 1;
            if (!mbar_wait(smem_u32(s_full + b), (j >> 1) & 1, a.dev_error)) { ok = false; break; }
            tc_fence_after();
            float sv[kN];
            {
                uint32_t raw[32];
#pragma unroll
                for (int q = 0; q < kN / 32; ++q) {
                    tmem_ld32(lane_base + (b ? C::kColS1 : C::kColS0) + q * 32, raw);
                    tc_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) sv[q * 32 + e] = __uint_as_float(raw[e]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(s_free + b));

            const int key0 = j * kN;
            float mt = -INFINITY;
            if (key0 + kN - 1 <= lim) {
#pragma unroll
                for (int e = 0; e < kN; ++e) {
                    sv[e] *= a.scale_log2;
                    mt = fmaxf(mt, sv[e]);
                }
            } else {
#pragma unroll
                for (int e = 0; e < kN; ++e) {
                    sv[e] = (key0 + e <= lim) ? sv[e] * a.scale_log2 : -INFINITY;
                    mt = fmaxf(mt, sv[e]);
                }
            }
            bool rescale = false;
            float corr = 1.f;
            if (mt > m_ref + 8.f) {                     // also true while m_ref is -inf
                corr = fast_exp2(m_ref - mt);
                m_ref = mt;
                rescale = true;
            }
            l *= corr;
            uint32_t pk[kN / 2];
#pragma unroll
            for (int e = 0; e < kN; e += 2) {
                const float p0 = fast_exp2(sv[e] - m_ref);
                const float p1 = fast_exp2(sv[e + 1] - m_ref);
                pk[e / 2] = pack_bf16(p0, p1);
                const __nv_bfloat162 pb = *reinterpret_cast<const __nv_bfloat162 *>(&pk[e / 2]);
                l += __low2float(pb) + __high2float(pb);
            }
            // the previous PV product must be done before P and O are touched
            if (j >= 1 && !mbar_wait(smem_u32(pv_done), (j - 1) & 1, a.dev_error)) { ok = false; break; }
            if (rescale && j >= 1) {
                tc_fence_after();
#pragma unroll
                for (int q = 0; q < D / 32; ++q) {
                    uint32_t o[32];
                    tmem_ld32(lane_base + C::kColO + q * 32, o);
                    tc_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
                    tmem_st32(lane_base + C::kColO + q * 32, o);
                }
                tc_wait_st();
            }
#pragma unroll
            for (int kc = 0; kc < kN / 8; ++kc) {
                const uint32_t dst = p_s + (kc >> 3) * kSlab + swz128(r, kc & 7);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(pk[kc * 4]),
                             "r"(pk[kc * 4 + 1]), "r"(pk[kc * 4 + 2]), "r"(pk[kc * 4 + 3])
                             : "memory");
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(p_full));
        }
        // ---- epilogue: O / l -> bf16 rows ----
        if (ok && nkt > 0 && mbar_wait(smem_u32(pv_done), (nkt - 1) & 1, a.dev_error)) {
            tc_fence_after();
            const float inv = 1.f / l;
            const bool store = t < n_new;
            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out) +
                                                   ((int64_t)(q0 + (store ? t : 0)) * a.num_q_heads +
                                                    (int64_t)kvh * G + r % G) * D);
#pragma unroll
            for (int q = 0; q < D / 32; ++q) {
                uint32_t o[32];
                tmem_ld32(lane_base + C::kColO + q * 32, o);
                tc_wait_ld();
                if (store) {
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint4 v;
                        v.x = pack_bf16(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv);
                        v.y = pack_bf16(__uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
                        v.z = pack_bf16(__uint_as_float(o[e + 4]) * inv, __uint_as_float(o[e + 5]) * inv);
                        v.w = pack_bf16(__uint_as_float(o[e + 6]) * inv, __uint_as_float(o[e + 7]) * inv);
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
cudaError_t launch_prefill_d(const PrefillArgs &a, const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                             cudaStream_t stream) {
    using C = PrefillCfg<D>;
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = uint64_t(1) << (dev & 63);
    if (!(configured.load(std::memory_order_acquire) & bit)) {
        e = cudaFuncSetAttribute(prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
        if (e != cudaSuccess) return e;
        configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    const int TQ = kM / a.group;
    const dim3 grid((unsigned)(a.batch * a.num_kv_heads), (unsigned)((a.max_seqlen_q + TQ - 1) / TQ));
    prefill_kernel<D><<<grid, kThreads, C::kSmemBytes, stream>>>(tm_k, tm_v, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs &a, const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                           cudaStream_t stream) {
    if (a.head_dim == 128) return launch_prefill_d<128>(a, tm_k, tm_v, stream);
    return launch_prefill_d<64>(a, tm_k, tm_v, stream);
}

}  // namespace pa
