"""Thin ctypes binding over libpagedattn.so, with the C ABI's names.

Argument marshalling only: every step of the hot path runs in the CUDA
kernels behind the C ABI (include/pa.h).  There is no CPU or PyTorch fallback:
if the library is missing or a call fails, these functions raise.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedattn.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "pa.h")

_lib = None
_lock = threading.Lock()

PA_OK = 0
PA_ERR_INVALID_ARG = 1
PA_ERR_UNSUPPORTED = 2
PA_ERR_CUDA = 3
PA_ERR_DEVICE_CHECK = 4
PA_ERR_TIMEOUT = 5
PA_ERR_WORKSPACE = 6

PA_DEVERR_BLOCK_ID = 0x1
PA_DEVERR_SLOT = 0x2
PA_DEVERR_CONTEXT_LEN = 0x4
PA_DEVERR_SEQLENS = 0x8
PA_DEVERR_TIMEOUT = 0x10

__all__ = ["PagedAttnError", "load_library", "declared_symbols", "pa_store_kv", "pa_decode", "pa_decode_split",
           "pa_store_kv_decode", "pa_store_kv_prefill_varlen", "pa_prefill_varlen_mixed",
           "pa_prefill_varlen_mixed_workspace_size", "alloc_mixed_workspace",
           "pa_decode_workspace_size", "pa_decode_split_workspace_size", "pa_decode_noalloc",
           "pa_decode_shared_prefix", "pa_decode_shared_prefix_workspace_size", "alloc_shared_prefix_workspace", "pa_prefill_varlen",
           "pa_prefill_workspace_size", "pa_selftest_bounded_wait", "pa_selftest_exp2", "pa_status_string",
           "pa_version",
           "alloc_decode_workspace", "alloc_prefill_workspace"]


class PagedAttnError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        super().__init__(f"{pa_status_string(status)}: {detail}")


_c_i32, _c_i64, _c_f32, _c_sz, _c_p = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p

_SIGS = {
    "pa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "pa_last_error_detail": (ctypes.c_char_p, []),
    "pa_version": (ctypes.c_int, []),
    "pa_store_kv": (ctypes.c_int, [_c_p, _c_p, _c_i64, _c_i64, _c_p, _c_i32, _c_p, _c_p, _c_i32, _c_i32, _c_i32,
                                   _c_i32, _c_p, _c_p]),
    "pa_decode_workspace_size": (_c_sz, [_c_i32] * 6),
    "pa_decode_split_workspace_size": (_c_sz, [_c_i32] * 6),
    "pa_decode": (ctypes.c_int, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_i32, _c_p, _c_i32, _c_i32, _c_i32, _c_i32,
                                 _c_i32, _c_i32, _c_i32, _c_f32, _c_p, _c_sz, _c_p, _c_p]),
    "pa_store_kv_decode": (ctypes.c_int, [_c_p, _c_p, _c_i64, _c_i64, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_i32,
                                          _c_p, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_f32, _c_p,
                                          _c_sz, _c_p, _c_p]),
    "pa_decode_split": (ctypes.c_int, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_i32, _c_p, _c_i32, _c_i32, _c_i32, _c_i32,
                                       _c_i32, _c_i32, _c_i32, _c_f32, _c_i32, _c_p, _c_sz, _c_p, _c_p]),
    "pa_decode_shared_prefix_workspace_size": (_c_sz, [_c_i32] * 7),
    "pa_decode_shared_prefix": (ctypes.c_int, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_i32, _c_p, _c_i32, _c_i32, _c_i32,
                                               _c_i32, _c_i32, _c_i32, _c_i32, _c_f32, _c_i32, _c_p, _c_sz, _c_p,
                                               _c_p]),
    "pa_decode_noalloc_max_scratch_bytes": (_c_sz, []),
    "pa_decode_noalloc": (ctypes.c_int, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_i32, _c_p, _c_i32, _c_i32, _c_i32, _c_i32,
                                         _c_i32, _c_i32, _c_i32, _c_f32, _c_p, _c_p]),
    "pa_prefill_workspace_size": (_c_sz, [_c_i32] * 5),
    "pa_prefill_varlen": (ctypes.c_int, [_c_p, _c_p, _c_i32, _c_p, _c_p, _c_p, _c_p, _c_i32, _c_i32, _c_p, _c_i32, _c_i32,
                                         _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_f32, _c_i32, _c_p, _c_sz, _c_p,
                                         _c_p]),
    "pa_store_kv_prefill_varlen": (ctypes.c_int, [_c_p, _c_p, _c_i64, _c_i64, _c_p, _c_p, _c_p, _c_i32, _c_p, _c_p,
                                                  _c_p, _c_p, _c_i32, _c_i32, _c_p, _c_i32, _c_i32, _c_i32, _c_i32,
                                                  _c_i32, _c_i32, _c_i32, _c_f32, _c_i32, _c_p, _c_sz, _c_p, _c_p]),
    "pa_prefill_varlen_mixed_workspace_size": (_c_sz, [_c_i32] * 6),
    "pa_prefill_varlen_mixed": (ctypes.c_int, [_c_p, _c_p, _c_i32, _c_p, _c_p, _c_p, _c_p, _c_i32, _c_i32, _c_p,
                                               _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_f32, _c_p,
                                               _c_sz, _c_p, _c_p]),
    "pa_selftest_bounded_wait": (ctypes.c_int, [_c_p, _c_i64, _c_p]),
    "pa_selftest_exp2": (ctypes.c_int, [_c_p, _c_p, _c_p, _c_i32, _c_p]),
}


def declared_symbols():
    """Names of every entry point include/pa.h declares."""
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^PA_API\s+[\w\s\*]*?\b(pa_\w+)\s*\(", txt, flags=re.M)))


def load_library():
    """Load libpagedattn.so (raises if it is not built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m paged_kv_cache_325_b200.build` (nvcc, sm_100a)")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in _SIGS.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def pa_status_string(status: int) -> str:
    return load_library().pa_status_string(int(status)).decode()


def pa_version() -> int:
    return int(load_library().pa_version())


def _check(status: int):
    if status != PA_OK:
        raise PagedAttnError(status, load_library().pa_last_error_detail().decode())


# ------------------------------------------------------------ marshalling --

def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(t, stream):
    import torch
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype=None, device=None, contiguous=True):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _cache_dims(k_cache, v_cache):
    import torch
    _need(k_cache, "k_cache", torch.bfloat16)
    _need(v_cache, "v_cache", torch.bfloat16, k_cache.device)
    if k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("k_cache/v_cache must both be [num_blocks, block_size, num_kv_heads, head_dim]")
    return tuple(int(x) for x in k_cache.shape)


def _opt_err(dev_error, device):
    import torch
    if dev_error is not None:
        _need(dev_error, "dev_error", torch.int32, device)
    return _ptr(dev_error)


def pa_store_kv(k, v, slot_mapping, k_cache, v_cache, dev_error=None, stream=None):
    """Write k[i], v[i] into cache slot slot_mapping[i] (rows with a negative slot are skipped)."""
    import torch
    nb, B, Hkv, D = _cache_dims(k_cache, v_cache)
    dev = k_cache.device
    for name, t in (("k", k), ("v", v)):
        _need(t, name, torch.bfloat16, dev, contiguous=False)
        if t.dim() != 3 or tuple(t.shape[1:]) != (Hkv, D) or t.stride(2) != 1 or t.stride(1) != D:
            raise ValueError(f"{name} must be [N, num_kv_heads, head_dim] with contiguous rows")
    _need(slot_mapping, "slot_mapping", torch.int32, dev)
    n = int(slot_mapping.shape[0])
    if k.shape[0] != n or v.shape[0] != n:
        raise ValueError("k, v and slot_mapping must have the same number of rows")
    _check(load_library().pa_store_kv(_ptr(k), _ptr(v), k.stride(0), v.stride(0), _ptr(slot_mapping), n,
                                      _ptr(k_cache), _ptr(v_cache), nb, B, Hkv, D, _opt_err(dev_error, dev),
                                      _stream(k_cache, stream)))


def pa_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, block_size) -> int:
    return int(load_library().pa_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim,
                                                       max_context_len, block_size))


def pa_decode_split_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, num_splits) -> int:
    return int(load_library().pa_decode_split_workspace_size(batch, num_q_heads, num_kv_heads, head_dim,
                                                             max_context_len, num_splits))


def alloc_decode_workspace(q, num_kv_heads, max_context_len, block_size, num_splits=0):
    """A torch-owned workspace of the size pa_decode (num_splits=0) or pa_decode_split needs."""
    import torch
    batch, Hq, D = q.shape
    if num_splits:
        n = pa_decode_split_workspace_size(batch, Hq, num_kv_heads, D, max_context_len, num_splits)
    else:
        n = pa_decode_workspace_size(batch, Hq, num_kv_heads, D, max_context_len, block_size)
    return torch.empty(max(n, 1), dtype=torch.uint8, device=q.device)


def _decode_args(out, q, k_cache, v_cache, block_table, context_lens):
    import torch
    nb, B, Hkv, D = _cache_dims(k_cache, v_cache)
    dev = k_cache.device
    _need(q, "q", torch.bfloat16, dev)
    _need(out, "out", torch.bfloat16, dev)
    if q.dim() != 3 or q.shape[2] != D or out.shape != q.shape:
        raise ValueError("q and out must be [batch, num_q_heads, head_dim]")
    _need(block_table, "block_table", torch.int32, dev)
    _need(context_lens, "context_lens", torch.int32, dev)
    batch, Hq, _ = q.shape
    if block_table.dim() != 2 or block_table.shape[0] != batch or context_lens.shape != (batch,):
        raise ValueError("block_table must be [batch, max_blocks] and context_lens [batch]")
    return nb, B, Hkv, D, batch, Hq, dev


def pa_decode(out, q, k_cache, v_cache, block_table, context_lens, max_context_len, softmax_scale,
              workspace=None, dev_error=None, stream=None, num_splits=None):
    """Paged GQA decode attention into `out` ([batch, Hq, D] bf16)."""
    nb, B, Hkv, D, batch, Hq, dev = _decode_args(out, q, k_cache, v_cache, block_table, context_lens)
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if workspace is not None:
        _need(workspace, "workspace", None, dev)
    lib = load_library()
    common = (_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), block_table.shape[1],
              _ptr(context_lens), batch, int(max_context_len), Hq, Hkv, D, nb, B, float(softmax_scale))
    if num_splits is None:
        st = lib.pa_decode(*common, _ptr(workspace), ws, _opt_err(dev_error, dev), _stream(q, stream))
    else:
        st = lib.pa_decode_split(*common, int(num_splits), _ptr(workspace), ws, _opt_err(dev_error, dev),
                                 _stream(q, stream))
    _check(st)


def pa_store_kv_decode(k, v, slot_mapping, out, q, k_cache, v_cache, block_table, context_lens, max_context_len,
                       softmax_scale, workspace=None, dev_error=None, stream=None):
    """pa_store_kv of this step's rows (row s = sequence s's new token) and pa_decode, in one launch."""
    import torch
    nb, B, Hkv, D, batch, Hq, dev = _decode_args(out, q, k_cache, v_cache, block_table, context_lens)
    for name, t in (("k", k), ("v", v)):
        _need(t, name, torch.bfloat16, dev, contiguous=False)
        if t.dim() != 3 or tuple(t.shape) != (batch, Hkv, D) or t.stride(2) != 1 or t.stride(1) != D:
            raise ValueError(f"{name} must be [batch, num_kv_heads, head_dim] with contiguous rows")
    _need(slot_mapping, "slot_mapping", torch.int32, dev)
    if tuple(slot_mapping.shape) != (batch,):
        raise ValueError("slot_mapping must be [batch]")
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if workspace is not None:
        _need(workspace, "workspace", None, dev)
    _check(load_library().pa_store_kv_decode(
        _ptr(k), _ptr(v), k.stride(0), v.stride(0), _ptr(slot_mapping), _ptr(out), _ptr(q), _ptr(k_cache),
        _ptr(v_cache), _ptr(block_table), block_table.shape[1], _ptr(context_lens), batch, int(max_context_len), Hq,
        Hkv, D, nb, B, float(softmax_scale), _ptr(workspace), ws, _opt_err(dev_error, dev), _stream(q, stream)))


def pa_decode_split(out, q, k_cache, v_cache, block_table, context_lens, max_context_len, softmax_scale,
                    num_splits, workspace=None, dev_error=None, stream=None):
    """pa_decode with an explicit number of context splits (0 = automatic)."""
    pa_decode(out, q, k_cache, v_cache, block_table, context_lens, max_context_len, softmax_scale,
              workspace=workspace, dev_error=dev_error, stream=stream, num_splits=num_splits)


def pa_decode_shared_prefix_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, block_size,
                                           num_shared_blocks) -> int:
    return int(load_library().pa_decode_shared_prefix_workspace_size(batch, num_q_heads, num_kv_heads, head_dim,
                                                                      max_context_len, block_size, num_shared_blocks))


def alloc_shared_prefix_workspace(q, num_kv_heads, max_context_len, block_size, num_shared_blocks):
    import torch
    batch, Hq, D = q.shape
    n = pa_decode_shared_prefix_workspace_size(batch, Hq, num_kv_heads, D, max_context_len, block_size,
                                               num_shared_blocks)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)


def pa_decode_shared_prefix(out, q, k_cache, v_cache, block_table, context_lens, max_context_len, softmax_scale,
                            num_shared_blocks, workspace, dev_error=None, stream=None):
    """Decode for a batch whose block tables all start with the same num_shared_blocks blocks."""
    nb, B, Hkv, D, batch, Hq, dev = _decode_args(out, q, k_cache, v_cache, block_table, context_lens)
    _need(workspace, "workspace", None, dev)
    _check(load_library().pa_decode_shared_prefix(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), block_table.shape[1],
        _ptr(context_lens), batch, int(max_context_len), Hq, Hkv, D, nb, B, float(softmax_scale),
        int(num_shared_blocks), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _opt_err(dev_error, dev), _stream(q, stream)))


def pa_decode_noalloc(out, q, k_cache, v_cache, block_table, context_lens, max_context_len, softmax_scale,
                      dev_error=None, stream=None):
    """pa_decode without a workspace: the split scratch is the library's fixed per-GPU array."""
    nb, B, Hkv, D, batch, Hq, dev = _decode_args(out, q, k_cache, v_cache, block_table, context_lens)
    _check(load_library().pa_decode_noalloc(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), block_table.shape[1],
        _ptr(context_lens), batch, int(max_context_len), Hq, Hkv, D, nb, B, float(softmax_scale),
        _opt_err(dev_error, dev), _stream(q, stream)))


def pa_prefill_workspace_size(batch, max_seqlen_q, num_q_heads, num_kv_heads, head_dim) -> int:
    return int(load_library().pa_prefill_workspace_size(batch, max_seqlen_q, num_q_heads, num_kv_heads, head_dim))


def alloc_prefill_workspace(q, num_kv_heads, batch, max_seqlen_q):
    """A torch-owned workspace of the size pa_prefill_varlen needs (its work-unit table)."""
    import torch
    n = pa_prefill_workspace_size(batch, max_seqlen_q, q.shape[1], num_kv_heads, q.shape[2])
    return torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)


def pa_prefill_varlen(out, q, k_cache, v_cache, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                      block_table, softmax_scale, causal=True, workspace=None, dev_error=None, stream=None):
    """Varlen (causal) prefill over the paged cache into `out` ([total_q, Hq, D] bf16).

    `workspace`: device scratch of pa_prefill_workspace_size() bytes (alloc_prefill_workspace)."""
    import torch
    nb, B, Hkv, D = _cache_dims(k_cache, v_cache)
    dev = k_cache.device
    _need(q, "q", torch.bfloat16, dev)
    _need(out, "out", torch.bfloat16, dev)
    if q.dim() != 3 or q.shape[2] != D or out.shape != q.shape:
        raise ValueError("q and out must be [total_q, num_q_heads, head_dim]")
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32, dev)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32, dev)
    _need(block_table, "block_table", torch.int32, dev)
    batch = int(cu_seqlens_q.shape[0]) - 1
    if cu_seqlens_k.shape != cu_seqlens_q.shape or block_table.dim() != 2 or block_table.shape[0] != batch:
        raise ValueError("cu_seqlens_q/k must be [batch+1] and block_table [batch, max_blocks]")
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load_library().pa_prefill_varlen(
        _ptr(out), _ptr(q), int(q.shape[0]), _ptr(k_cache), _ptr(v_cache), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
        int(max_seqlen_q), int(max_seqlen_k), _ptr(block_table), block_table.shape[1], batch, q.shape[1], Hkv, D,
        nb, B, float(softmax_scale), int(bool(causal)), _ptr(workspace), ws, _opt_err(dev_error, dev),
        _stream(q, stream)))


def pa_store_kv_prefill_varlen(k, v, slot_mapping, out, q, k_cache, v_cache, cu_seqlens_q, cu_seqlens_k,
                               max_seqlen_q, max_seqlen_k, block_table, softmax_scale, causal=True, workspace=None,
                               dev_error=None, stream=None):
    """pa_store_kv of the prompts' new rows and pa_prefill_varlen in one launch, the new keys read from k / v."""
    import torch
    nb, B, Hkv, D = _cache_dims(k_cache, v_cache)
    dev = k_cache.device
    _need(q, "q", torch.bfloat16, dev)
    _need(out, "out", torch.bfloat16, dev)
    if q.dim() != 3 or q.shape[2] != D or out.shape != q.shape:
        raise ValueError("q and out must be [total_q, num_q_heads, head_dim]")
    total_q = int(q.shape[0])
    for name, t in (("k", k), ("v", v)):
        _need(t, name, torch.bfloat16, dev, contiguous=False)
        if t.dim() != 3 or tuple(t.shape) != (total_q, Hkv, D) or t.stride(2) != 1 or t.stride(1) != D:
            raise ValueError(f"{name} must be [total_q, num_kv_heads, head_dim] with contiguous rows")
    _need(slot_mapping, "slot_mapping", torch.int32, dev)
    if tuple(slot_mapping.shape) != (total_q,):
        raise ValueError("slot_mapping must be [total_q]")
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32, dev)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32, dev)
    _need(block_table, "block_table", torch.int32, dev)
    batch = int(cu_seqlens_q.shape[0]) - 1
    if cu_seqlens_k.shape != cu_seqlens_q.shape or block_table.dim() != 2 or block_table.shape[0] != batch:
        raise ValueError("cu_seqlens_q/k must be [batch+1] and block_table [batch, max_blocks]")
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load_library().pa_store_kv_prefill_varlen(
        _ptr(k), _ptr(v), k.stride(0), v.stride(0), _ptr(slot_mapping), _ptr(out), _ptr(q), total_q, _ptr(k_cache),
        _ptr(v_cache), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), int(max_seqlen_q), int(max_seqlen_k),
        _ptr(block_table), block_table.shape[1], batch, q.shape[1], Hkv, D, nb, B, float(softmax_scale),
        int(bool(causal)), _ptr(workspace), ws, _opt_err(dev_error, dev), _stream(q, stream)))


def pa_prefill_varlen_mixed_workspace_size(batch, max_seqlen_q, max_seqlen_k, num_q_heads, num_kv_heads,
                                           head_dim) -> int:
    return int(load_library().pa_prefill_varlen_mixed_workspace_size(batch, max_seqlen_q, max_seqlen_k, num_q_heads,
                                                                     num_kv_heads, head_dim))


def alloc_mixed_workspace(q, num_kv_heads, batch, max_seqlen_q, max_seqlen_k):
    """A torch-owned workspace of the size pa_prefill_varlen_mixed needs."""
    import torch
    n = pa_prefill_varlen_mixed_workspace_size(batch, max_seqlen_q, max_seqlen_k, q.shape[1], num_kv_heads,
                                               q.shape[2])
    return torch.empty(max(n, 1), dtype=torch.uint8, device=q.device)


def pa_prefill_varlen_mixed(out, q, k_cache, v_cache, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                            block_table, softmax_scale, workspace=None, dev_error=None, stream=None):
    """Causal varlen attention for a batch mixing prompts and decode steps (one-token sequences go to the
    decode kernel, the rest to the prefill kernel)."""
    import torch
    nb, B, Hkv, D = _cache_dims(k_cache, v_cache)
    dev = k_cache.device
    _need(q, "q", torch.bfloat16, dev)
    _need(out, "out", torch.bfloat16, dev)
    if q.dim() != 3 or q.shape[2] != D or out.shape != q.shape:
        raise ValueError("q and out must be [total_q, num_q_heads, head_dim]")
    _need(cu_seqlens_q, "cu_seqlens_q", torch.int32, dev)
    _need(cu_seqlens_k, "cu_seqlens_k", torch.int32, dev)
    _need(block_table, "block_table", torch.int32, dev)
    batch = int(cu_seqlens_q.shape[0]) - 1
    if cu_seqlens_k.shape != cu_seqlens_q.shape or block_table.dim() != 2 or block_table.shape[0] != batch:
        raise ValueError("cu_seqlens_q/k must be [batch+1] and block_table [batch, max_blocks]")
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load_library().pa_prefill_varlen_mixed(
        _ptr(out), _ptr(q), int(q.shape[0]), _ptr(k_cache), _ptr(v_cache), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
        int(max_seqlen_q), int(max_seqlen_k), _ptr(block_table), block_table.shape[1], batch, q.shape[1], Hkv, D,
        nb, B, float(softmax_scale), _ptr(workspace), ws, _opt_err(dev_error, dev), _stream(q, stream)))


def pa_selftest_bounded_wait(dev_error, max_polls, stream=None):
    """Run the bounded-wait self-test kernel; it ORs PA_DEVERR_TIMEOUT into dev_error."""
    import torch
    _need(dev_error, "dev_error", torch.int32)
    _check(load_library().pa_selftest_bounded_wait(_ptr(dev_error), int(max_polls), _stream(dev_error, stream)))


def pa_selftest_exp2(x, stream=None):
    """Evaluate the prefill softmax's two exponentials on a float32 CUDA tensor x: returns (y_poly, y_sfu)."""
    import torch
    _need(x, "x", dtype=torch.float32)
    y_poly, y_sfu = torch.empty_like(x), torch.empty_like(x)
    _check(load_library().pa_selftest_exp2(_ptr(x), _ptr(y_poly), _ptr(y_sfu), x.numel(), _stream(x, stream)))
    return y_poly, y_sfu
