"""pa_store_kv_decode (store_kvcache inside the paged decode's launch), and the
merge of the decode's context splits whatever the workspace held before, on the
GPU against the fp64 oracle.

The oracle runs its own store, then its decode, on the same seeded bytes; the
cache the fused call leaves behind must equal the oracle's stored cache bit for
bit, and the output must meet the attention tolerance.  Cache slots no context
covers, and the new tokens' slots before the store, hold bf16 NaN, so a decode
that read the cache row instead of the new token would return NaN.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_325_b200 as pa
from paged_kv_cache_325_b200 import workloads as W
from gpu_helpers import DecodeOnGpu, assert_close, i32, oracle_decode

pytestmark = pytest.mark.gpu


def _fused(g, num_splits=None, dev_error=None, workspace=None, out=None):
    c = g.case
    ws = workspace if workspace is not None else pa.alloc_decode_workspace(g.q, c.num_kv_heads, c.max_context_len,
                                                                           c.block_size)
    out = torch.empty_like(g.q) if out is None else out
    pa.pa_store_kv_decode(g.k_new, g.v_new, g.slot_mapping, out, g.q, g.k_cache, g.v_cache, g.block_table,
                          g.context_lens, c.max_context_len, c.softmax_scale, workspace=ws, dev_error=dev_error)
    return out


def _cache_equals_oracle_store(g, case):
    kc, vc = oracle.store(case.k_new, case.v_new, case.slot_mapping, case.k_cache, case.v_cache)
    assert torch.equal(g.k_cache.cpu().view(torch.int16), kc.view(torch.int16)), "k_cache differs from the store"
    assert torch.equal(g.v_cache.cpu().view(torch.int16), vc.view(torch.int16)), "v_cache differs from the store"


@pytest.mark.parametrize("make", [W.tiny_decode, W.qwen3_06b_decode, W.long_context_decode],
                         ids=["tiny", "qwen3_0.6b", "long_context"])
def test_store_decode_workloads(cuda_lib, make):
    case = make()
    g = DecodeOnGpu(case)
    out = _fused(g)
    torch.cuda.synchronize()
    assert_close(out, oracle_decode(case), what=case.name)
    _cache_equals_oracle_store(g, case)


@pytest.mark.parametrize("ctx", [[1200] + [64] * 60, [6000] + [64] * 100], ids=["few_splits", "many_splits"])
def test_store_decode_skewed_batch_auto_splits(cuda_lib, ctx):
    """Store fused into a decode whose plan splits the long pair (merged in the kernel, or by the combine):
    the long sequence's CTA starts on its first tile before the plan exists, the short ones (one tile,
    which holds their new token) do not."""
    case = W.make_decode_case(ctx, 8, 2, 128, 64, seed=1610 + len(ctx))
    g = DecodeOnGpu(case)
    out = _fused(g)
    torch.cuda.synchronize()
    assert_close(out, oracle_decode(case), what=f"{len(ctx)} sequences")
    _cache_equals_oracle_store(g, case)


@pytest.mark.parametrize("B", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("Hq,Hkv,D", [(8, 4, 128), (32, 8, 64), (6, 1, 64), (16, 16, 128)])
def test_store_decode_shapes(cuda_lib, B, Hq, Hkv, D):
    # contexts that put the new token first, last and in the middle of a tile, a warp slice and a block
    ctx = [1, 2, 16, 17, 63, 64, 65, 100, B, B + 1, 3 * B - 1, 700]
    case = W.make_decode_case(ctx, Hq, Hkv, D, B, seed=1600 + B + Hq + D)
    g = DecodeOnGpu(case)
    out = _fused(g)
    torch.cuda.synchronize()
    assert_close(out, oracle_decode(case), what=f"B={B} Hq={Hq} Hkv={Hkv} D={D}")
    _cache_equals_oracle_store(g, case)


def test_store_decode_matches_separate_calls_bitwise(cuda_lib):
    """Same launch geometry, same arithmetic: fused and store-then-decode agree bit for bit."""
    case = W.make_decode_case([5, 300, 1024, 2000, 77], 16, 4, 128, 64, seed=1701)
    g1, g2 = DecodeOnGpu(case), DecodeOnGpu(case)
    out1 = _fused(g1)
    g2.store()
    out2 = g2.decode()
    torch.cuda.synchronize()
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    assert torch.equal(g1.k_cache.view(torch.int16), g2.k_cache.view(torch.int16))


def test_store_decode_padding_rows(cuda_lib):
    """slot_mapping = -1 rows store nothing; their decode reads the cache as it is."""
    case = W.make_decode_case([40, 300, 129, 64], 8, 2, 128, 16, seed=1702, poison=False)
    slots = case.slot_mapping.copy()
    slots[1] = -1
    slots[3] = -1
    case.slot_mapping = slots
    g = DecodeOnGpu(case)
    out = _fused(g)
    torch.cuda.synchronize()
    assert_close(out, oracle_decode(case), what="padding rows")
    _cache_equals_oracle_store(g, case)


def test_store_decode_checked_mode(cuda_lib):
    case = W.make_decode_case([40, 300, 129], 8, 2, 128, 16, seed=1703, poison=False)
    err = torch.zeros(1, dtype=torch.int32, device="cuda:0")
    g = DecodeOnGpu(case)
    _fused(g, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    # a slot other than the new token's position is reported (and still written, as pa_store_kv would)
    other = case.slot_mapping.copy()
    other[1] = (other[1] + 1) % (case.num_blocks * case.block_size)
    g = DecodeOnGpu(case)
    g.slot_mapping = i32(other, g.dev)
    _fused(g, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pa.PA_DEVERR_SLOT
    kc, _ = oracle.store(case.k_new, case.v_new, other, case.k_cache, case.v_cache)
    assert torch.equal(g.k_cache.cpu().view(torch.int16), kc.view(torch.int16))
    # a slot past the cache is reported and not written
    err.zero_()
    bad = case.slot_mapping.copy()
    bad[0] = case.num_blocks * case.block_size + 5
    g = DecodeOnGpu(case)
    g.slot_mapping = i32(bad, g.dev)
    _fused(g, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pa.PA_DEVERR_SLOT
    skipped = case.slot_mapping.copy()
    skipped[0] = -1
    kc, vc = oracle.store(case.k_new, case.v_new, skipped, case.k_cache, case.v_cache)
    assert torch.equal(g.k_cache.cpu().view(torch.int16), kc.view(torch.int16))
    assert torch.equal(g.v_cache.cpu().view(torch.int16), vc.view(torch.int16))


def test_store_decode_stores_rows_of_rejected_sequences(cuda_lib):
    """A sequence whose context length is rejected (0, or past max_context_len) gets no decode, but its
    new row is still stored, as pa_store_kv then pa_decode would leave the cache; the other sequences'
    outputs are unaffected and the rejected sequences' output rows are left as they were."""
    case = W.make_decode_case([40, 300, 129, 77], 8, 2, 128, 16, seed=1707, poison=False)
    ctx = case.context_lens.copy()
    ctx[1] = 0                              # invalid: below 1
    ctx[3] = case.max_context_len + 50      # invalid: past max_context_len
    g = DecodeOnGpu(case)
    g.context_lens = i32(ctx, g.dev)
    err = torch.zeros(1, dtype=torch.int32, device=g.dev)
    out = torch.full_like(g.q, 7.0)
    _fused(g, dev_error=err, out=out)
    torch.cuda.synchronize()
    assert int(err.item()) & pa.PA_DEVERR_CONTEXT_LEN
    _cache_equals_oracle_store(g, case)
    ref = oracle_decode(case)
    for s in (0, 2):
        assert_close(out[s], ref[s], what=f"valid sequence {s}")
    for s in (1, 3):
        assert bool((out[s] == 7.0).all()), f"output of rejected sequence {s} was written"


def test_store_decode_rejects_unaligned_rows(cuda_lib):
    case = W.tiny_decode()
    g = DecodeOnGpu(case)
    wide = torch.zeros(case.batch, case.num_kv_heads * case.head_dim + 4, dtype=torch.bfloat16, device=g.dev)
    k = wide[:, :case.num_kv_heads * case.head_dim].view(case.batch, case.num_kv_heads, case.head_dim)
    with pytest.raises(pa.PagedAttnError) as e:
        pa.pa_store_kv_decode(k, g.v_new, g.slot_mapping, torch.empty_like(g.q), g.q, g.k_cache, g.v_cache,
                              g.block_table, g.context_lens, case.max_context_len, case.softmax_scale,
                              workspace=pa.alloc_decode_workspace(g.q, case.num_kv_heads, case.max_context_len,
                                                                  case.block_size))
    assert e.value.status == pa.PA_ERR_UNSUPPORTED


# ---------------------------------------------------------------- merge --

def test_split_merge_ignores_workspace_contents(cuda_lib):
    """The split partials live in the workspace; whatever it holds beforehand (random bytes, zeros, all
    ones, the leftovers of a call with another shape) must not change the result."""
    case = W.make_decode_case([3000, 777, 4100, 64, 2500, 1], 32, 8, 128, 256, seed=1704)
    g = DecodeOnGpu(case)
    g.store()
    torch.cuda.synchronize()
    ref = oracle_decode(case)
    n = pa.pa_decode_workspace_size(case.batch, 32, 8, 128, case.max_context_len, 256)
    gen = torch.Generator(device="cpu").manual_seed(5)
    for fill in ("random", "zeros", "ones", "other_shape"):
        ws = torch.empty(n + 4096, dtype=torch.uint8, device=g.dev)
        if fill == "random":
            ws.copy_(torch.randint(0, 256, (ws.numel(),), dtype=torch.uint8, generator=gen))
        elif fill == "zeros":
            ws.zero_()
        elif fill == "ones":
            ws.fill_(255)
        else:
            other = W.make_decode_case([100, 5000, 2048], 16, 4, 128, 256, seed=1705)
            go = DecodeOnGpu(other)
            go.store()
            ws2 = ws[:pa.pa_decode_workspace_size(3, 16, 4, 128, other.max_context_len, 256)]
            pa.pa_decode(torch.empty_like(go.q), go.q, go.k_cache, go.v_cache, go.block_table, go.context_lens,
                         other.max_context_len, other.softmax_scale, workspace=ws2)
        for rep in range(2):                 # and again on what this call left behind
            out = torch.empty_like(g.q)
            pa.pa_decode(out, g.q, g.k_cache, g.v_cache, g.block_table, g.context_lens, case.max_context_len,
                         case.softmax_scale, workspace=ws[:n])
            torch.cuda.synchronize()
            assert_close(out, ref, what=f"workspace {fill} rep {rep}")


def test_shared_prefix_sequence_without_private_tokens(cuda_lib):
    """A shared-prefix sequence whose context ends exactly at the shared blocks has no private split;
    the merge covers its prefix chunks alone."""
    B, P = 16, 3
    case = W.make_decode_case([P * B + 1, P * B + 40, P * B + 1], 8, 2, 128, B, seed=1706,
                              shared_prefix_blocks=P, poison=False)
    g = DecodeOnGpu(case)
    g.store()
    ctx = case.context_lens.copy()
    ctx[0] = P * B                      # sequence 0 sees the shared blocks only
    g.context_lens = i32(ctx, g.dev)
    mcl = case.max_context_len
    ws = pa.alloc_shared_prefix_workspace(g.q, case.num_kv_heads, mcl, B, P)
    out = torch.empty_like(g.q)
    pa.pa_decode_shared_prefix(out, g.q, g.k_cache, g.v_cache, g.block_table, g.context_lens, mcl,
                               case.softmax_scale, P, ws)
    torch.cuda.synchronize()
    kc, vc = oracle.store(case.k_new, case.v_new, case.slot_mapping, case.k_cache, case.v_cache)
    ref = oracle.decode(case.q, kc, vc, case.block_table, ctx, case.softmax_scale)
    assert_close(out, ref, what="empty private split")
