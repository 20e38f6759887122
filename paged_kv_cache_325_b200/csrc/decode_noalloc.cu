// pa_decode_noalloc: pa_decode for callers that cannot allocate device memory.
//
// Some callers have no way to obtain device scratch: a plugin or embedded
// runtime whose host application owns every device allocation, or an engine
// that has handed all spare HBM to its KV-cache pool and keeps no allocator
// on the decode path.  For them this entry point takes its split-KV scratch
// from a fixed array compiled into the library instead of a caller workspace.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds kNoAllocScratchBytes of it until the process exits.  Host code
// must not pass the variable's name to a kernel (on the host that name is a
// stand-in, not a device address).  Every call asks the runtime for the
// array's address on the current device (cudaGetSymbolAddress, a table lookup
// once the module is loaded) instead of keeping it: after a cudaDeviceReset,
// or any other teardown of the context, the module is loaded again and the
// array may sit elsewhere, so a kept address could point at freed memory.
#include <cuda_runtime.h>

#include "pa.h"
#include "pa_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // 8 MiB per device

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

// Device address of g_decode_scratch in the current device's context.
pa_status scratch_for_current_device(void **out) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || !p) {
        pa::set_last_error(PA_ERR_CUDA, "pa_decode_noalloc: cudaGetSymbolAddress of the static scratch failed");
        return PA_ERR_CUDA;
    }
    *out = p;
    return PA_OK;
}

}  // namespace

extern "C" {

size_t pa_decode_noalloc_max_scratch_bytes(void) { return kNoAllocScratchBytes; }

pa_status pa_decode_noalloc(void *out, const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *block_table, int32_t block_table_stride, const int32_t *context_lens,
                            int32_t batch, int32_t max_context_len, int32_t num_q_heads, int32_t num_kv_heads,
                            int32_t head_dim, int32_t num_blocks, int32_t block_size, float softmax_scale,
                            int32_t *dev_error, void *stream) {
    const size_t need = pa_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                                 block_size);
    if (need > kNoAllocScratchBytes) {
        pa::set_last_error(PA_ERR_WORKSPACE,
                           "pa_decode_noalloc: these sizes need more split scratch than the library's fixed "
                           "array holds; use pa_decode with a caller workspace");
        return PA_ERR_WORKSPACE;
    }
    void *scratch = nullptr;
    if (need > 0) {
        pa_status st = scratch_for_current_device(&scratch);
        if (st != PA_OK) return st;
    }
    return pa_decode(out, q, k_cache, v_cache, block_table, block_table_stride, context_lens, batch,
                     max_context_len, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size, softmax_scale,
                     scratch, need > 0 ? kNoAllocScratchBytes : 0, dev_error, stream);
}

}  // extern "C"
