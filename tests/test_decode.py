"""pa_decode on the GPU against the fp64 oracle (store then decode, same bytes).

Tolerance: max-abs 1e-2 and mean-abs 1e-3 over all outputs.  Cache slots that
no context covers hold bf16 NaN, so any read past a context shows up as a
non-finite output.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_325_b200 as pa
from paged_kv_cache_325_b200 import workloads as W
from gpu_helpers import DecodeOnGpu, assert_close, i32, oracle_decode

pytestmark = pytest.mark.gpu


def _run(case, num_splits=None):
    g = DecodeOnGpu(case)
    g.store()
    out = g.decode(num_splits=num_splits)
    torch.cuda.synchronize()
    return g, out


@pytest.mark.parametrize("make", [W.tiny_decode, W.qwen3_06b_decode, W.long_context_decode,
                                  W.prefix_sharing_decode],
                         ids=["tiny", "qwen3_0.6b", "long_context", "prefix_sharing"])
def test_decode_workloads_full_size(cuda_lib, make):
    case = make()
    _, out = _run(case)
    ref = oracle_decode(case)
    assert_close(out, ref, what=case.name)


@pytest.mark.parametrize("ctx,what", [
    # one long context among short ones: the long pairs are cut into chunks plus four smaller tail pieces
    # (7 splits: merged inside the decode kernel by the CTA that finishes the last one) ...
    ([1200] + [64] * 60, "merged in the decode kernel"),
    # ... and with many splits per pair (14: merged by the combine kernel); fewer (sequence, KV head) pairs
    # than CTAs, so most CTAs start on the counter instead of a pair of their own
    ([6000] + [64] * 100, "merged by the combine kernel"),
])
def test_decode_skewed_batch_auto_splits(cuda_lib, ctx, what):
    case = W.make_decode_case(ctx, 8, 2, 128, 64, seed=310 + len(ctx))
    _, out = _run(case)
    assert_close(out, oracle_decode(case), what=what)


@pytest.mark.parametrize("num_splits", [1, 2, 3, 5, 16])
def test_decode_explicit_splits(cuda_lib, num_splits):
    case = W.make_decode_case([1, 63, 64, 65, 200, 511, 777, 1024], 8, 2, 128, 64, seed=300 + num_splits)
    _, out = _run(case, num_splits=num_splits)
    assert_close(out, oracle_decode(case), what=f"splits={num_splits}")


@pytest.mark.parametrize("B", [16, 32, 64, 128, 256])
def test_decode_block_sizes(cuda_lib, B):
    case = W.make_decode_case([1, 15, 16, 17, 130, 257, 600], 8, 4, 128, B, seed=400 + B)
    for splits in (None, 3):
        _, out = _run(case, num_splits=splits)
        assert_close(out, oracle_decode(case), what=f"B={B} splits={splits}")


@pytest.mark.parametrize("Hq,Hkv,D", [(4, 4, 128), (16, 8, 128), (32, 8, 64), (16, 2, 128), (32, 2, 64),
                                      (12, 4, 128), (6, 1, 64)])
def test_decode_gqa_groups_and_head_dims(cuda_lib, Hq, Hkv, D):
    case = W.make_decode_case([5, 99, 300, 1000], Hq, Hkv, D, 16, seed=500 + Hq * 7 + Hkv + D)
    for splits in (None, 4):
        _, out = _run(case, num_splits=splits)
        assert_close(out, oracle_decode(case), what=f"Hq={Hq} Hkv={Hkv} D={D} splits={splits}")


def test_decode_context_one_returns_v_exactly(cuda_lib):
    case = W.make_decode_case([1] * 6, 8, 2, 128, 16, seed=601)
    _, out = _run(case)
    G = 4
    want = case.v_new.repeat_interleave(G, dim=1)
    assert torch.equal(out.cpu().view(torch.int16), want.view(torch.int16))


def test_decode_block_relabelling_is_bitwise_invariant(cuda_lib):
    case = W.make_decode_case([40, 300, 1000], 8, 2, 128, 16, seed=602)
    _, a = _run(case, num_splits=3)
    rng = np.random.default_rng(9)
    pi = rng.permutation(case.num_blocks).astype(np.int32)
    kc = torch.empty_like(case.k_cache)
    vc = torch.empty_like(case.v_cache)
    kc[torch.from_numpy(pi).long()] = case.k_cache
    vc[torch.from_numpy(pi).long()] = case.v_cache
    bt = case.block_table.copy()
    bt[bt >= 0] = pi[bt[bt >= 0]]
    case.k_cache, case.v_cache, case.block_table = kc, vc, bt
    case.slot_mapping = np.array([pi[s // 16] * 16 + s % 16 for s in case.slot_mapping], dtype=np.int32)
    _, b = _run(case, num_splits=3)
    assert torch.equal(a.cpu().view(torch.int16), b.cpu().view(torch.int16))


def test_decode_max_context_len_above_actual(cuda_lib):
    case = W.make_decode_case([10, 20, 30], 4, 2, 64, 16, seed=603)
    g = DecodeOnGpu(case)
    g.store()
    out = g.decode(max_context_len=4096)
    torch.cuda.synchronize()
    assert_close(out, oracle_decode(case), what="max_context_len 4096")


def test_decode_checked_mode_flags_bad_inputs(cuda_lib):
    dev = torch.device("cuda:0")
    case = W.make_decode_case([10, 20, 30], 4, 2, 64, 16, seed=604)
    g = DecodeOnGpu(case)
    g.store()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    g.decode(dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    bad = case.block_table.copy()
    bad[1, 0] = case.num_blocks + 5                       # block id past the pool
    g.block_table = i32(bad, dev)
    g.decode(dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pa.PA_DEVERR_BLOCK_ID
    g.block_table = i32(case.block_table, dev)
    err.zero_()
    g.context_lens = i32([10, 0, 30], dev)                # empty context
    g.decode(dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pa.PA_DEVERR_CONTEXT_LEN
    err.zero_()
    g.context_lens = i32([10, 20, 31], dev)               # longer than max_context_len
    g.decode(dev_error=err, max_context_len=30)
    torch.cuda.synchronize()
    assert int(err.item()) & pa.PA_DEVERR_CONTEXT_LEN


def test_decode_workspace_too_small_is_rejected(cuda_lib):
    case = W.make_decode_case([3000, 4000], 8, 2, 128, 256, seed=605)
    g = DecodeOnGpu(case)
    small = torch.empty(16, dtype=torch.uint8, device=g.dev)
    with pytest.raises(pa.PagedAttnError) as ei:
        pa.pa_decode(g.out, g.q, g.k_cache, g.v_cache, g.block_table, g.context_lens, 4000, case.softmax_scale,
                     workspace=small, num_splits=4)
    assert ei.value.status == pa.PA_ERR_WORKSPACE


def test_bounded_wait_self_test_reports_timeout(cuda_lib):
    dev = torch.device("cuda:0")
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    pa.pa_selftest_bounded_wait(err, 1000)
    torch.cuda.synchronize()
    assert int(err.item()) & pa.PA_DEVERR_TIMEOUT
    # the context is still usable
    case = W.tiny_decode()
    _, out = _run(case)
    assert_close(out, oracle_decode(case), what="after timeout self-test")
