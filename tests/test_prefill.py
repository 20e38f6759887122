"""pa_prefill_varlen on the GPU against the fp64 oracle (store then prefill).

Tolerance: max-abs 1e-2 and mean-abs 1e-3.  Cache slots no context covers
hold bf16 NaN; the new tokens' slots are NaN until pa_store_kv writes them.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_325_b200 as pa
from paged_kv_cache_325_b200 import workloads as W
from gpu_helpers import (MAX_ABS, MEAN_ABS, PrefillOnGpu, assert_close, bf16_half_ulp, i32, oracle_prefill,
                         varlen_prefill_reference)

pytestmark = pytest.mark.gpu


def _run(case, causal=None):
    g = PrefillOnGpu(case)
    g.store()
    out = g.prefill(causal=causal)
    torch.cuda.synchronize()
    return g, out


def test_prefill_varlen_workload_every_row(cuda_lib):
    """The full-size varlen prefill workload (12 prompts up to 2048 tokens, half with a cached prefix),
    every element of every (new token, q-head) row against the oracle."""
    case, ref = varlen_prefill_reference()
    _, out = _run(case)
    assert_close(out, ref, what="varlen_prefill, every row")


@pytest.mark.parametrize("B", [16, 32, 64, 128, 256])
def test_prefill_block_sizes_with_cached_prefix(cuda_lib, B):
    L = [1, 40, 2 * B + 5, 3 * B, 300]
    c = [0, 0, B, 2 * B, (300 - 1) // B * B]
    case = W.make_prefill_case(L, c, 8, 2, 128, B, seed=700 + B)
    _, out = _run(case)
    assert_close(out, oracle_prefill(case), what=f"B={B}")


@pytest.mark.parametrize("Hq,Hkv,D", [(8, 8, 128), (16, 8, 64), (32, 8, 128), (16, 2, 128), (32, 2, 64),
                                      (16, 1, 128), (4, 4, 64)])
def test_prefill_gqa_groups_and_head_dims(cuda_lib, Hq, Hkv, D):
    case = W.make_prefill_case([7, 33, 129, 260], [0, 16, 64, 128], Hq, Hkv, D, 16, seed=800 + Hq + Hkv + D)
    _, out = _run(case)
    assert_close(out, oracle_prefill(case), what=f"Hq={Hq} Hkv={Hkv} D={D}")


@pytest.mark.parametrize("n_new", [1, 31, 32, 33, 127, 128, 129, 500])
def test_prefill_tile_edges(cuda_lib, n_new):
    case = W.make_prefill_case([n_new, n_new + 256], [0, 256], 32, 8, 128, 256, seed=900 + n_new)
    _, out = _run(case)
    assert_close(out, oracle_prefill(case), what=f"n_new={n_new}")


def test_prefill_non_causal(cuda_lib):
    case = W.make_prefill_case([50, 300], [0, 128], 16, 4, 128, 64, seed=951, causal=False)
    _, out = _run(case)
    assert_close(out, oracle_prefill(case), what="non-causal")


def test_prefill_sequence_with_no_new_tokens(cuda_lib):
    case = W.make_prefill_case([64, 100, 37], [64, 0, 32], 8, 2, 128, 32, seed=952)
    assert int(case.cu_seqlens_q[1] - case.cu_seqlens_q[0]) == 0
    _, out = _run(case)
    assert_close(out, oracle_prefill(case), what="empty sequence in batch")


def test_prefill_row_matches_gpu_decode(cuda_lib):
    """The prefill row of a new token at position t-1 equals decode with context t."""
    case = W.make_prefill_case([300], [256], 16, 4, 128, 16, seed=953)
    g, out = _run(case)
    n_new = 300 - 256
    ctx = [256 + i + 1 for i in range(n_new)]
    q = g.q.clone()
    dout = torch.empty_like(q)
    bt = g.block_table.repeat(n_new, 1)
    pa.pa_decode(dout, q, g.k_cache, g.v_cache, bt, i32(ctx, g.dev), 300, case.softmax_scale,
                 workspace=pa.alloc_decode_workspace(q, 4, 300, 16))
    torch.cuda.synchronize()
    a, b = out.double().cpu().numpy(), dout.double().cpu().numpy()
    diff = np.abs(a - b)
    # both sides are rounded to bf16: allow one ulp of the output on top of the bar
    assert (diff - 2 * bf16_half_ulp(b)).max() <= MAX_ABS and diff.mean() <= MEAN_ABS


def test_prefill_checked_mode(cuda_lib):
    case = W.make_prefill_case([40, 70], [32, 0], 8, 2, 64, 16, seed=954)
    g = PrefillOnGpu(case)
    g.store()
    err = torch.zeros(1, dtype=torch.int32, device=g.dev)
    g.prefill(dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    bad = case.block_table.copy()
    bad[1, 2] = -7
    g.block_table = i32(bad, g.dev)
    g.prefill(dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pa.PA_DEVERR_BLOCK_ID
    err.zero_()
    g.block_table = i32(case.block_table, g.dev)
    g.cu_k = i32([0, 5, 75], g.dev)                      # n_k < n_new for sequence 0
    g.prefill(dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pa.PA_DEVERR_SEQLENS


def test_prefill_many_sequences_exercise_persistent_units(cuda_lib):
    """Far more work units than SMs: every CTA walks many units, carrying its
    barrier phases and TMEM buffers from one unit to the next."""
    rng = np.random.default_rng(31)
    L = rng.integers(1, 400, size=180)
    c = np.array([(int(x) - 1) // 64 * 64 if i % 3 == 0 else 0 for i, x in enumerate(L)])
    case = W.make_prefill_case(L, c, 16, 4, 128, 64, seed=961)
    _, out = _run(case)
    assert_close(out, oracle_prefill(case), what="180 sequences")


def test_prefill_head_dim_64_long_prompt(cuda_lib):
    case = W.make_prefill_case([1500, 700], [1024, 0], 32, 8, 64, 256, seed=962)
    _, out = _run(case)
    assert_close(out, oracle_prefill(case), what="D=64 long prompt, every row")
