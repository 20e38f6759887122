"""pa_decode_shared_prefix on the GPU: the prefix-sharing decode path (shared
blocks read once per KV head, private suffixes by split-KV decode, partials
merged by log-sum-exp) against the fp64 oracle, which gathers every sequence's
whole context independently."""
import numpy as np
import pytest
import torch

import paged_kv_cache_325_b200 as pa
from paged_kv_cache_325_b200 import workloads as W
from gpu_helpers import DecodeOnGpu, assert_close, i32, oracle_decode

pytestmark = pytest.mark.gpu


def _run(case, P, dev_error=None, max_context_len=None):
    g = DecodeOnGpu(case)
    g.store()
    mcl = int(max_context_len or case.max_context_len)
    ws = pa.alloc_shared_prefix_workspace(g.q, case.num_kv_heads, mcl, case.block_size, P)
    out = torch.empty_like(g.q)
    pa.pa_decode_shared_prefix(out, g.q, g.k_cache, g.v_cache, g.block_table, g.context_lens, mcl,
                               case.softmax_scale, P, ws, dev_error=dev_error)
    torch.cuda.synchronize()
    return g, out


def test_shared_prefix_workload_full_size(cuda_lib):
    case = W.prefix_sharing_decode()
    _, out = _run(case, 16)
    assert_close(out, oracle_decode(case), what="prefix_sharing")


@pytest.mark.parametrize("Hq,Hkv,D,B,P", [(16, 8, 128, 256, 2), (8, 2, 128, 16, 5), (16, 4, 64, 64, 3),
                                          (32, 8, 128, 32, 9), (4, 4, 64, 16, 1)])
def test_shared_prefix_shapes(cuda_lib, Hq, Hkv, D, B, P):
    rng = np.random.default_rng(Hq + 7 * P + B)
    ctx = P * B + 1 + rng.integers(0, 300, size=37)
    ctx[0] = P * B + 1                     # only the new token is private
    case = W.make_decode_case(ctx, Hq, Hkv, D, B, seed=1300 + P, shared_prefix_blocks=P)
    _, out = _run(case, P)
    assert_close(out, oracle_decode(case), what=f"Hq={Hq} Hkv={Hkv} D={D} B={B} P={P}")


def test_shared_prefix_matches_plain_decode(cuda_lib):
    case = W.make_decode_case(4096 + 1 + np.arange(40) * 13, 16, 8, 128, 256, seed=1401, shared_prefix_blocks=16)
    g, out = _run(case, 16)
    ref = g.decode()
    torch.cuda.synchronize()
    a, b = out.double().cpu().numpy(), ref.double().cpu().numpy()
    from gpu_helpers import MAX_ABS, MEAN_ABS, bf16_half_ulp
    diff = np.abs(a - b)
    assert (diff - 2 * bf16_half_ulp(b)).max() <= MAX_ABS and diff.mean() <= MEAN_ABS


def test_shared_prefix_checked_mode(cuda_lib):
    case = W.make_decode_case([70, 90, 100], 8, 2, 128, 16, seed=1402, shared_prefix_blocks=4)
    err = torch.zeros(1, dtype=torch.int32, device="cuda:0")
    _run(case, 4, dev_error=err)
    assert int(err.item()) == 0
    bad = case.block_table.copy()
    bad[2, 1] = bad[0, 5]                    # row 2 no longer shares block 1 of the prefix
    case.block_table = bad
    _run(case, 4, dev_error=err)
    assert int(err.item()) & pa.PA_DEVERR_BLOCK_ID
