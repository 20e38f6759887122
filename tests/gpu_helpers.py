"""Shared helpers of the GPU parity tests: run a workload through the C ABI and
through the CPU oracle on the same seeded bytes, and compare."""
import functools

import numpy as np
import torch

import oracle
import paged_kv_cache_325_b200 as pa

# Tolerance of the attention outputs against the fp64 oracle (bf16 in, fp32
# accumulate, bf16 out): max-abs 1e-2 and mean-abs 1e-3.  The output itself is
# bf16, whose rounding alone is up to half an ulp (2^-9 relative; 0.0156 for
# |x| in [4, 8)), so the max-abs bar applies to the error beyond that rounding:
# |gpu - ref| <= 1e-2 + ulp_bf16(ref) / 2 elementwise.
MAX_ABS = 1e-2
MEAN_ABS = 1e-3


def i32(a, dev):
    return torch.as_tensor(np.ascontiguousarray(a, dtype=np.int32)).to(dev)


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers at |x| (8 significant bits)."""
    _, e = np.frexp(np.abs(x))                # |x| = m * 2^e, m in [0.5, 1)
    return np.where(x == 0, 0.0, np.ldexp(1.0, e - 9))


def assert_close(gpu_bf16: torch.Tensor, ref: np.ndarray, max_abs=MAX_ABS, mean_abs=MEAN_ABS, what=""):
    g = gpu_bf16.detach().to("cpu", torch.float64).numpy().reshape(ref.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite GPU output"
    err = np.abs(g - ref)
    excess = err - bf16_half_ulp(ref)
    assert excess.max() <= max_abs, (f"{what}: error beyond bf16 output rounding {excess.max():.3e} > {max_abs} "
                                     f"(raw max abs {err.max():.3e})")
    assert err.mean() <= mean_abs, f"{what}: mean abs err {err.mean():.3e} > {mean_abs}"
    return float(err.max()), float(err.mean())


class DecodeOnGpu:
    """A decode case resident on the GPU (cache copied before the store)."""

    def __init__(self, case, dev="cuda:0"):
        self.case = case
        self.dev = torch.device(dev)
        self.k_cache = case.k_cache.to(self.dev)
        self.v_cache = case.v_cache.to(self.dev)
        self.k_new = case.k_new.to(self.dev)
        self.v_new = case.v_new.to(self.dev)
        self.q = case.q.to(self.dev)
        self.slot_mapping = i32(case.slot_mapping, self.dev)
        self.block_table = i32(case.block_table, self.dev)
        self.context_lens = i32(case.context_lens, self.dev)
        self.out = torch.empty_like(self.q)

    def store(self, dev_error=None):
        pa.pa_store_kv(self.k_new, self.v_new, self.slot_mapping, self.k_cache, self.v_cache, dev_error=dev_error)

    def decode(self, num_splits=None, dev_error=None, max_context_len=None, out=None):
        c = self.case
        mcl = int(max_context_len or c.max_context_len)
        ws = pa.alloc_decode_workspace(self.q, c.num_kv_heads, mcl, c.block_size, num_splits or 0)
        out = self.out if out is None else out
        pa.pa_decode(out, self.q, self.k_cache, self.v_cache, self.block_table, self.context_lens, mcl,
                     c.softmax_scale, workspace=ws, dev_error=dev_error, num_splits=num_splits)
        return out


def oracle_decode(case, seq_idx=None, head_idx=None):
    kc, vc = oracle.store(case.k_new, case.v_new, case.slot_mapping, case.k_cache, case.v_cache)
    return oracle.decode(case.q, kc, vc, case.block_table, case.context_lens, case.softmax_scale,
                         seq_idx=seq_idx, head_idx=head_idx)


class PrefillOnGpu:
    def __init__(self, case, dev="cuda:0"):
        self.case = case
        self.dev = torch.device(dev)
        self.k_cache = case.k_cache.to(self.dev)
        self.v_cache = case.v_cache.to(self.dev)
        self.k_new = case.k_new.to(self.dev)
        self.v_new = case.v_new.to(self.dev)
        self.q = case.q.to(self.dev)
        self.slot_mapping = i32(case.slot_mapping, self.dev)
        self.block_table = i32(case.block_table, self.dev)
        self.cu_q = i32(case.cu_seqlens_q, self.dev)
        self.cu_k = i32(case.cu_seqlens_k, self.dev)
        self.out = torch.empty_like(self.q)
        self.ws = pa.alloc_prefill_workspace(self.q, case.num_kv_heads, case.batch, max(1, case.max_seqlen_q))

    def store(self, dev_error=None):
        pa.pa_store_kv(self.k_new, self.v_new, self.slot_mapping, self.k_cache, self.v_cache, dev_error=dev_error)

    def prefill(self, dev_error=None, causal=None):
        c = self.case
        pa.pa_prefill_varlen(self.out, self.q, self.k_cache, self.v_cache, self.cu_q, self.cu_k, c.max_seqlen_q,
                             c.max_seqlen_k, self.block_table, c.softmax_scale,
                             causal=c.causal if causal is None else causal, workspace=self.ws, dev_error=dev_error)
        return self.out


def oracle_prefill(case, tok_idx=None, head_idx=None, causal=None):
    kc, vc = oracle.store(case.k_new, case.v_new, case.slot_mapping, case.k_cache, case.v_cache)
    return oracle.prefill(case.q, kc, vc, case.cu_seqlens_q, case.cu_seqlens_k, case.block_table,
                          case.softmax_scale, causal=case.causal if causal is None else causal,
                          tok_idx=tok_idx, head_idx=head_idx)


@functools.lru_cache(maxsize=1)
def varlen_prefill_reference():
    """The full-size varlen prefill workload (poisoned parity form) and the oracle's result for every
    (new token, q-head) row; computed once per test session (about 10 s of fp64 on 16 threads)."""
    from paged_kv_cache_325_b200 import workloads as W
    case = W.varlen_prefill()
    return case, oracle_prefill(case)
