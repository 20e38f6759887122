// store_kvcache: scatter this step's new K/V rows into the block-paged cache.
//
// One warp per token row.  A row is num_kv_heads * head_dim bf16 values
// (2 KB for 8 KV heads of 128), copied with 16-byte vector loads and stores by
// the 32 lanes of the warp, K then V.  The operation is the slot_mapping
// write of the nano-vllm walkthrough (xingyun3d.csdn.net, section seven) and
// the Triton store kernel of the gitcode.csdn.net nano-vLLM article (section
// 3.4); it is a pure copy, bit-exact by construction.
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr int kStoreWarpsPerBlock = 8;

template <bool kVec16>
__global__ void __launch_bounds__(kStoreWarpsPerBlock * 32)
    store_kv_kernel(const StoreArgs a) {
    const int lane = threadIdx.x & 31;
    const int64_t i = (int64_t)blockIdx.x * kStoreWarpsPerBlock + (threadIdx.x >> 5);
    if (i >= a.num_tokens) return;
    const int64_t slot = __ldg(a.slot_mapping + i);
    if (slot < 0) return;                       // padding row: nothing to store
    if (slot >= a.num_slots) {                  // never write outside the cache
        if (lane == 0) report(a.dev_error, PA_DEVERR_SLOT);
        return;
    }
    const uint16_t *ks = static_cast<const uint16_t *>(a.k) + i * a.k_row_stride;
    const uint16_t *vs = static_cast<const uint16_t *>(a.v) + i * a.v_row_stride;
    uint16_t *kd = static_cast<uint16_t *>(a.k_cache) + slot * a.row_elems;
    uint16_t *vd = static_cast<uint16_t *>(a.v_cache) + slot * a.row_elems;
    if constexpr (kVec16) {
        const int n16 = a.row_elems / 8;
        const uint4 *k4 = reinterpret_cast<const uint4 *>(ks);
        const uint4 *v4 = reinterpret_cast<const uint4 *>(vs);
        uint4 *kd4 = reinterpret_cast<uint4 *>(kd);
        uint4 *vd4 = reinterpret_cast<uint4 *>(vd);
        // issue every load of the row before the stores, so each lane has
        // several 16-byte requests in flight
        constexpr int kMaxPerLane = 8;          // rows up to 8 * 32 * 16 B = 4 KB in one pass
        for (int base = 0; base < n16; base += 32 * kMaxPerLane) {
            uint4 kr[kMaxPerLane], vr[kMaxPerLane];
#pragma unroll
            for (int u = 0; u < kMaxPerLane; ++u) {
                const int c = base + u * 32 + lane;
                if (c < n16) {
                    kr[u] = __ldg(k4 + c);
                    vr[u] = __ldg(v4 + c);
                }
            }
#pragma unroll
            for (int u = 0; u < kMaxPerLane; ++u) {
                const int c = base + u * 32 + lane;
                if (c < n16) {
                    kd4[c] = kr[u];
                    vd4[c] = vr[u];
                }
            }
        }
    } else {
        for (int c = lane; c < a.row_elems; c += 32) {
            kd[c] = ks[c];
            vd[c] = vs[c];
        }
    }
}

}  // namespace

cudaError_t launch_store(const StoreArgs &a, cudaStream_t stream) {
    if (a.num_tokens == 0) return cudaSuccess;
    const bool vec = ((reinterpret_cast<uintptr_t>(a.k) | reinterpret_cast<uintptr_t>(a.v)) % 16 == 0) &&
                     (a.k_row_stride % 8 == 0) && (a.v_row_stride % 8 == 0) && (a.row_elems % 8 == 0);
    const dim3 grid((unsigned)((a.num_tokens + kStoreWarpsPerBlock - 1) / kStoreWarpsPerBlock));
    if (vec)
        store_kv_kernel<true><<<grid, kStoreWarpsPerBlock * 32, 0, stream>>>(a);
    else
        store_kv_kernel<false><<<grid, kStoreWarpsPerBlock * 32, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace pa
