"""CPU fp64 oracle for the paged-KV hot path (ctypes wrapper over pa_oracle.c).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
(``paged_kv_cache_325_b200``) never imports it, and it imports nothing from that
library: the two share no code.  The only thing both sides consume is the
seeded input generator, which holds no attention arithmetic.

Every entry follows the definition written out at the top of pa_oracle.c:
gather each sequence's K/V through its block table, then softmax(q K^T *
scale) V with the GQA head mapping h -> h // (Hq / Hkv), in double precision.
Parity status: every function here is pinned by tests/test_oracle.py (brute
force, closed forms, invariants and a library cross-check); none is unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_I32P = ctypes.POINTER(ctypes.c_int32)
_U16P = ctypes.POINTER(ctypes.c_uint16)
_F64P = ctypes.POINTER(ctypes.c_double)
_lock = threading.Lock()
_default = None


def compile_oracle(src: str, out: str) -> str:
    """Compile an oracle C source with gcc (OpenMP, strict IEEE double arithmetic)."""
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-std=c11", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Build liboracle.so next to pa_oracle.c if it is missing or stale."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        compile_oracle(_SRC, _LIB_PATH)
    return _LIB_PATH


class Oracle:
    """One loaded copy of the oracle library (the default one, or a test's mutant)."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        lib.oracle_store.restype = ctypes.c_int
        lib.oracle_store.argtypes = [_U16P, _U16P, ctypes.c_int64, ctypes.c_int64, _I32P, ctypes.c_int32,
                                     _U16P, _U16P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32]
        lib.oracle_decode.restype = ctypes.c_int
        lib.oracle_decode.argtypes = [_F64P, ctypes.c_int32, _I32P, _I32P, _U16P, _U16P, _U16P, _I32P,
                                      ctypes.c_int32, _I32P, ctypes.c_int32, ctypes.c_int32,
                                      ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                      ctypes.c_double]
        lib.oracle_prefill.restype = ctypes.c_int
        lib.oracle_prefill.argtypes = [_F64P, ctypes.c_int32, _I32P, _I32P, _U16P, _U16P, _U16P, _I32P,
                                       _I32P, _I32P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                       ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                       ctypes.c_double, ctypes.c_int32]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        self.lib = lib

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    def store(self, k, v, slot_mapping, k_cache, v_cache):
        """Return new (k_cache, v_cache) with rows slot_mapping[i] >= 0 replaced by k[i], v[i]."""
        kb, vb = _bits(k), _bits(v)
        kc, vc = _bits(k_cache).copy(), _bits(v_cache).copy()
        sm = _i32(slot_mapping)
        nb, B, Hkv, D = k_cache.shape
        rc = self.lib.oracle_store(_p(kb, _U16P), _p(vb, _U16P), Hkv * D, Hkv * D, _p(sm, _I32P), len(sm),
                                   _p(kc, _U16P), _p(vc, _U16P), nb * B, Hkv, D)
        if rc != 0:
            raise ValueError("oracle_store: slot out of range")
        to_t = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).reshape(k_cache.shape)
        return to_t(kc), to_t(vc)

    def store_inplace(self, k, v, slot_mapping, k_cache, v_cache):
        """The same row copy as store(), written into k_cache / v_cache themselves (contiguous CPU bf16
        tensors) instead of into fresh copies of them, so that timing it measures the scatter alone."""
        assert k_cache.is_contiguous() and v_cache.is_contiguous()
        kb, vb = _bits(k), _bits(v)
        kc = k_cache.view(torch.int16).numpy().view(np.uint16)
        vc = v_cache.view(torch.int16).numpy().view(np.uint16)
        sm = _i32(slot_mapping)
        nb, B, Hkv, D = k_cache.shape
        rc = self.lib.oracle_store(_p(kb, _U16P), _p(vb, _U16P), Hkv * D, Hkv * D, _p(sm, _I32P), len(sm),
                                   _p(kc, _U16P), _p(vc, _U16P), nb * B, Hkv, D)
        if rc != 0:
            raise ValueError("oracle_store: slot out of range")

    def decode(self, q, k_cache, v_cache, block_table, context_lens, softmax_scale, seq_idx=None,
               head_idx=None):
        """fp64 decode attention.  Returns [batch, Hq, D], or [len(seq_idx), D] for sampled pairs."""
        batch, Hq, D = q.shape
        nb, B, Hkv, _ = k_cache.shape
        bt = _i32(block_table)
        if bt.ndim == 1:
            bt = bt.reshape(batch, -1)
        ctx = _i32(context_lens)
        qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
        if seq_idx is None:
            nrows = batch * Hq
            si = hi = None
        else:
            si, hi = _i32(seq_idx), _i32(head_idx)
            nrows = len(si)
        out = np.empty((nrows, D), dtype=np.float64)
        rc = self.lib.oracle_decode(_p(out, _F64P), nrows, None if si is None else _p(si, _I32P),
                                    None if hi is None else _p(hi, _I32P), _p(qb, _U16P), _p(kb, _U16P),
                                    _p(vb, _U16P), _p(bt, _I32P), bt.shape[1], _p(ctx, _I32P), batch, Hq,
                                    Hkv, D, nb, B, float(softmax_scale))
        if rc != 0:
            raise ValueError("oracle_decode: index out of range")
        return out.reshape(batch, Hq, D) if seq_idx is None else out

    def prefill(self, q, k_cache, v_cache, cu_seqlens_q, cu_seqlens_k, block_table, softmax_scale,
                causal=True, tok_idx=None, head_idx=None):
        """fp64 varlen prefill.  Returns [total_q, Hq, D], or [len(tok_idx), D] for sampled rows."""
        total_q, Hq, D = q.shape
        nb, B, Hkv, _ = k_cache.shape
        cq, ck = _i32(cu_seqlens_q), _i32(cu_seqlens_k)
        bt = _i32(block_table)
        if bt.ndim == 1:
            bt = bt.reshape(len(cq) - 1, -1)
        qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
        if tok_idx is None:
            nrows = total_q * Hq
            ti = hi = None
        else:
            ti, hi = _i32(tok_idx), _i32(head_idx)
            nrows = len(ti)
        out = np.empty((nrows, D), dtype=np.float64)
        rc = self.lib.oracle_prefill(_p(out, _F64P), nrows, None if ti is None else _p(ti, _I32P),
                                     None if hi is None else _p(hi, _I32P), _p(qb, _U16P), _p(kb, _U16P),
                                     _p(vb, _U16P), _p(cq, _I32P), _p(ck, _I32P), _p(bt, _I32P), bt.shape[1],
                                     len(cq) - 1, Hq, Hkv, D, nb, B, float(softmax_scale),
                                     int(bool(causal)))
        if rc != 0:
            raise ValueError("oracle_prefill: index out of range")
        return out.reshape(total_q, Hq, D) if tok_idx is None else out


def default() -> Oracle:
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


def num_threads() -> int:
    return default().num_threads()


def store(*a, **kw):
    return default().store(*a, **kw)


def store_inplace(*a, **kw):
    return default().store_inplace(*a, **kw)


def decode(*a, **kw):
    return default().decode(*a, **kw)


def prefill(*a, **kw):
    return default().prefill(*a, **kw)


def _bits(t: torch.Tensor) -> np.ndarray:
    assert t.dtype == torch.bfloat16 and t.device.type == "cpu"
    return np.ascontiguousarray(t.contiguous().view(torch.int16).numpy()).view(np.uint16)


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _p(a: np.ndarray, typ):
    return a.ctypes.data_as(typ)
