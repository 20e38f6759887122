"""pa_prefill_varlen_mixed: one call for a batch that mixes decode steps (one new
token after a long cached context) with prompts (with and without a cached
prefix).  The one-token rows run in the decode kernel, the rest in the prefill
kernel; the result is the causal varlen attention the oracle computes for every
row.  Store first (pa_store_kv), then the call, as in the pages' step.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_325_b200 as pa
from paged_kv_cache_325_b200 import workloads as W
from gpu_helpers import MAX_ABS, MEAN_ABS, PrefillOnGpu, assert_close, bf16_half_ulp, oracle_prefill

pytestmark = pytest.mark.gpu


def _mixed(g, dev_error=None):
    c = g.case
    ws = pa.alloc_mixed_workspace(g.q, c.num_kv_heads, c.batch, c.max_seqlen_q, c.max_seqlen_k)
    out = torch.full_like(g.q, float("nan"))
    pa.pa_prefill_varlen_mixed(out, g.q, g.k_cache, g.v_cache, g.cu_q, g.cu_k, c.max_seqlen_q, c.max_seqlen_k,
                               g.block_table, c.softmax_scale, workspace=ws, dev_error=dev_error)
    return out


def _case(B, Hq, Hkv, D, seed):
    # decode steps (one new token after 1..40 cached blocks) interleaved with prompts
    rng = np.random.default_rng(seed)
    L, c = [], []
    for i in range(14):
        if i % 3 == 2:
            n = int(rng.integers(2, 300))
            pre = int(rng.integers(0, 3)) * B
            L.append(pre + n)
            c.append(pre)
        else:
            blocks = int(rng.integers(1, 41))
            L.append(blocks * B + 1)
            c.append(blocks * B)
    return W.make_prefill_case(L, c, Hq, Hkv, D, B, seed=seed)


@pytest.mark.parametrize("B,Hq,Hkv,D", [(16, 16, 4, 128), (256, 16, 4, 128), (64, 32, 8, 64), (32, 8, 8, 128)])
def test_mixed_batch_against_oracle(cuda_lib, B, Hq, Hkv, D):
    case = _case(B, Hq, Hkv, D, seed=2300 + B + Hq + D)
    g = PrefillOnGpu(case)
    g.store()
    out = _mixed(g)
    torch.cuda.synchronize()
    assert_close(out, oracle_prefill(case), what=f"mixed B={B} Hq={Hq} Hkv={Hkv} D={D}")


def test_mixed_batch_agrees_with_prefill_only(cuda_lib):
    """The same function as pa_prefill_varlen: prompt rows bit for bit (same kernel), decode rows within
    one output ulp plus the bar (other kernel, other rounding order)."""
    case = _case(64, 16, 4, 128, seed=2401)
    g = PrefillOnGpu(case)
    g.store()
    a = _mixed(g).clone()
    b = g.prefill().clone()
    torch.cuda.synchronize()
    n_new = np.diff(case.cu_seqlens_q)
    single = np.zeros(case.total_q, dtype=bool)
    for s in range(case.batch):
        if n_new[s] == 1:
            single[case.cu_seqlens_q[s]] = True
    single = torch.from_numpy(single).to(g.dev)
    assert torch.equal(a[~single].view(torch.int16), b[~single].view(torch.int16))
    x, y = a[single].double().cpu().numpy(), b[single].double().cpu().numpy()
    diff = np.abs(x - y)
    assert (diff - 2 * bf16_half_ulp(y)).max() <= MAX_ABS and diff.mean() <= MEAN_ABS


def test_mixed_batch_of_decode_rows_only(cuda_lib):
    L = [1 + 4 * 256, 1 + 30 * 256, 1 + 256, 1 + 120 * 256]
    case = W.make_prefill_case(L, [x - 1 for x in L], 32, 8, 128, 256, seed=2402)
    g = PrefillOnGpu(case)
    g.store()
    out = _mixed(g)
    torch.cuda.synchronize()
    assert_close(out, oracle_prefill(case), what="decode rows only")


def test_mixed_batch_of_prompts_only_is_the_prefill(cuda_lib):
    case = W.make_prefill_case([300, 77, 1000], [256, 0, 512], 32, 8, 128, 256, seed=2403)
    g = PrefillOnGpu(case)
    g.store()
    a = _mixed(g).clone()
    b = g.prefill().clone()
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_mixed_batch_checked_mode(cuda_lib):
    case = _case(16, 8, 2, 128, seed=2404)
    g = PrefillOnGpu(case)
    g.store()
    err = torch.zeros(1, dtype=torch.int32, device=g.dev)
    _mixed(g, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    bad = case.block_table.copy()
    bad[0, 0] = -3                            # sequence 0 is a decode row
    g.block_table = torch.as_tensor(bad).to(g.dev)
    _mixed(g, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pa.PA_DEVERR_BLOCK_ID
