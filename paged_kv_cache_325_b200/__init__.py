"""B200-native paged-KV hot path: store_kvcache, paged decode, varlen prefill.

The public calls carry the C ABI's names (include/pa.h) and are marshalled to
libpagedattn.so by ``_binding``; the library is loaded on first use.
"""
from ._binding import (  # noqa: F401
    PA_DEVERR_BLOCK_ID, PA_DEVERR_CONTEXT_LEN, PA_DEVERR_SEQLENS, PA_DEVERR_SLOT, PA_DEVERR_TIMEOUT,
    PA_ERR_CUDA, PA_ERR_DEVICE_CHECK, PA_ERR_INVALID_ARG, PA_ERR_TIMEOUT, PA_ERR_UNSUPPORTED, PA_ERR_WORKSPACE,
    PA_OK, PagedAttnError, alloc_decode_workspace, alloc_mixed_workspace, alloc_prefill_workspace, alloc_shared_prefix_workspace, declared_symbols, load_library, pa_decode, pa_decode_noalloc, pa_decode_shared_prefix, pa_decode_shared_prefix_workspace_size, pa_decode_split,
    pa_decode_split_workspace_size, pa_decode_workspace_size, pa_prefill_varlen, pa_prefill_varlen_mixed,
    pa_prefill_varlen_mixed_workspace_size, pa_prefill_workspace_size,
    pa_selftest_bounded_wait, pa_selftest_exp2, pa_status_string, pa_store_kv, pa_store_kv_decode, pa_store_kv_prefill_varlen, pa_version,
)
