"""pa_store_kv_prefill_varlen (store_kvcache of the prompts' new rows inside the
prefill launch, the new keys read straight from the new K/V rows) on the GPU
against the fp64 oracle, which runs its own store and then its prefill over the
cache.

Cache slots no context covers, and the new tokens' slots before the store, hold
bf16 NaN: a prefill that read a new key from the cache before the store would
return NaN, and the cache afterwards must equal the oracle's stored cache bit
for bit.  Tolerance: max-abs 1e-2 beyond the bf16 output rounding, mean-abs 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_325_b200 as pa
from paged_kv_cache_325_b200 import workloads as W
from gpu_helpers import PrefillOnGpu, assert_close, i32, oracle_prefill, varlen_prefill_reference

pytestmark = pytest.mark.gpu


def _fused(g, causal=None, dev_error=None, slots=None):
    c = g.case
    pa.pa_store_kv_prefill_varlen(g.k_new, g.v_new, g.slot_mapping if slots is None else slots, g.out, g.q,
                                  g.k_cache, g.v_cache, g.cu_q, g.cu_k, c.max_seqlen_q, c.max_seqlen_k,
                                  g.block_table, c.softmax_scale, causal=c.causal if causal is None else causal,
                                  workspace=g.ws, dev_error=dev_error)
    return g.out


def _cache_equals_oracle_store(g, case, slots=None):
    kc, vc = oracle.store(case.k_new, case.v_new, case.slot_mapping if slots is None else slots, case.k_cache,
                          case.v_cache)
    assert torch.equal(g.k_cache.cpu().view(torch.int16), kc.view(torch.int16)), "k_cache differs from the store"
    assert torch.equal(g.v_cache.cpu().view(torch.int16), vc.view(torch.int16)), "v_cache differs from the store"


def test_store_prefill_varlen_workload_every_row(cuda_lib):
    """The full-size varlen prefill workload with the store fused in: every element of every row against
    the oracle, and the cache bit for bit against the oracle's store."""
    case, ref = varlen_prefill_reference()
    g = PrefillOnGpu(case)
    out = _fused(g)
    torch.cuda.synchronize()
    assert_close(out, ref, what="varlen_prefill fused, every row")
    _cache_equals_oracle_store(g, case)


@pytest.mark.parametrize("B", [16, 32, 64, 128, 256])
def test_store_prefill_block_sizes_with_cached_prefix(cuda_lib, B):
    L = [1, 40, 2 * B + 5, 3 * B, 300]
    c = [0, 0, B, 2 * B, (300 - 1) // B * B]
    case = W.make_prefill_case(L, c, 8, 2, 128, B, seed=1800 + B)
    g = PrefillOnGpu(case)
    out = _fused(g)
    torch.cuda.synchronize()
    assert_close(out, oracle_prefill(case), what=f"B={B}")
    _cache_equals_oracle_store(g, case)


@pytest.mark.parametrize("Hq,Hkv,D", [(8, 8, 128), (16, 8, 64), (32, 8, 128), (16, 1, 128), (4, 4, 64)])
def test_store_prefill_gqa_groups_and_head_dims(cuda_lib, Hq, Hkv, D):
    case = W.make_prefill_case([7, 33, 129, 260], [0, 16, 64, 128], Hq, Hkv, D, 16, seed=1900 + Hq + Hkv + D)
    g = PrefillOnGpu(case)
    out = _fused(g)
    torch.cuda.synchronize()
    assert_close(out, oracle_prefill(case), what=f"Hq={Hq} Hkv={Hkv} D={D}")
    _cache_equals_oracle_store(g, case)


@pytest.mark.parametrize("n_new", [1, 31, 32, 33, 127, 128, 129, 500])
def test_store_prefill_tile_edges(cuda_lib, n_new):
    case = W.make_prefill_case([n_new, n_new + 256], [0, 256], 32, 8, 128, 256, seed=2100 + n_new)
    g = PrefillOnGpu(case)
    out = _fused(g)
    torch.cuda.synchronize()
    assert_close(out, oracle_prefill(case), what=f"n_new={n_new}")
    _cache_equals_oracle_store(g, case)


def test_store_prefill_non_causal(cuda_lib):
    case = W.make_prefill_case([50, 300], [0, 128], 16, 4, 128, 64, seed=2201, causal=False)
    g = PrefillOnGpu(case)
    out = _fused(g)
    torch.cuda.synchronize()
    assert_close(out, oracle_prefill(case), what="non-causal fused")
    _cache_equals_oracle_store(g, case)


def test_mixed_prefill_and_decode_rows(cuda_lib):
    """A mixed batch: sequences with one new token (decode steps, long cached contexts) beside prompts with
    and without a cached prefix, in one call.  The one-token rows must equal the decode of the same
    context."""
    B = 64
    L = [1 + 5 * B, 700, 1 + 12 * B, 90, 1 + 3 * B, 1 + B]
    c = [5 * B, 0, 12 * B, 0, 3 * B, B]
    case = W.make_prefill_case(L, c, 16, 4, 128, B, seed=2202)
    g = PrefillOnGpu(case)
    out = _fused(g)
    torch.cuda.synchronize()
    assert_close(out, oracle_prefill(case), what="mixed batch")
    _cache_equals_oracle_store(g, case)
    # the one-token rows through the decode kernel, on the cache the fused call left behind
    rows = [int(case.cu_seqlens_q[s]) for s in (0, 2, 4, 5)]
    q = g.q[torch.tensor(rows)].contiguous()
    bt = g.block_table[torch.tensor([0, 2, 4, 5])].contiguous()
    ctx = i32([L[s] for s in (0, 2, 4, 5)], g.dev)
    dout = torch.empty_like(q)
    pa.pa_decode(dout, q, g.k_cache, g.v_cache, bt, ctx, max(L), case.softmax_scale,
                 workspace=pa.alloc_decode_workspace(q, 4, max(L), B))
    torch.cuda.synchronize()
    from gpu_helpers import MAX_ABS, MEAN_ABS, bf16_half_ulp
    a, b = out[torch.tensor(rows)].double().cpu().numpy(), dout.double().cpu().numpy()
    diff = np.abs(a - b)
    assert (diff - 2 * bf16_half_ulp(b)).max() <= MAX_ABS and diff.mean() <= MEAN_ABS


def test_store_prefill_matches_separate_calls_bitwise(cuda_lib):
    """The same launch geometry and arithmetic: fused and store-then-prefill agree bit for bit."""
    case = W.make_prefill_case([300, 77, 1000], [256, 0, 512], 32, 8, 128, 256, seed=2203)
    g1, g2 = PrefillOnGpu(case), PrefillOnGpu(case)
    out1 = _fused(g1)
    g2.store()
    out2 = g2.prefill()
    torch.cuda.synchronize()
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    assert torch.equal(g1.k_cache.view(torch.int16), g2.k_cache.view(torch.int16))
    assert torch.equal(g1.v_cache.view(torch.int16), g2.v_cache.view(torch.int16))


def test_store_prefill_checked_mode(cuda_lib):
    case = W.make_prefill_case([40, 70], [32, 0], 8, 2, 64, 16, seed=2204, poison=False)
    err = torch.zeros(1, dtype=torch.int32, device="cuda:0")
    g = PrefillOnGpu(case)
    _fused(g, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    # a slot other than the token's position: reported, still written (as pa_store_kv would)
    other = case.slot_mapping.copy()
    other[3] = (other[3] + 1) % (case.num_blocks * case.block_size)
    g = PrefillOnGpu(case)
    _fused(g, dev_error=err, slots=i32(other, g.dev))
    torch.cuda.synchronize()
    assert int(err.item()) & pa.PA_DEVERR_SLOT
    _cache_equals_oracle_store(g, case, slots=other)
    # a negative slot and one past the cache: reported, not written
    err.zero_()
    bad = case.slot_mapping.copy()
    bad[0] = -1
    bad[5] = case.num_blocks * case.block_size + 3
    g = PrefillOnGpu(case)
    _fused(g, dev_error=err, slots=i32(bad, g.dev))
    torch.cuda.synchronize()
    assert int(err.item()) & pa.PA_DEVERR_SLOT
    skipped = bad.copy()
    skipped[5] = -1
    _cache_equals_oracle_store(g, case, slots=skipped)


def test_store_prefill_rejects_unaligned_rows(cuda_lib):
    case = W.make_prefill_case([40, 70], [32, 0], 8, 2, 64, 16, seed=2205)
    g = PrefillOnGpu(case)
    wide = torch.zeros(case.total_q, case.num_kv_heads * case.head_dim + 4, dtype=torch.bfloat16, device=g.dev)
    k = wide[:, :case.num_kv_heads * case.head_dim].view(case.total_q, case.num_kv_heads, case.head_dim)
    with pytest.raises(pa.PagedAttnError) as e:
        pa.pa_store_kv_prefill_varlen(k, g.v_new, g.slot_mapping, g.out, g.q, g.k_cache, g.v_cache, g.cu_q, g.cu_k,
                                      case.max_seqlen_q, case.max_seqlen_k, g.block_table, case.softmax_scale,
                                      workspace=g.ws)
    assert e.value.status == pa.PA_ERR_UNSUPPORTED
