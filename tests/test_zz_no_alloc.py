"""pa_decode_noalloc: the decode entry point for callers that cannot allocate
device memory (their host owns every allocation, or all spare HBM went to the
KV pool).  Its split scratch is a fixed array inside the library.

Calls the new entry point through the C ABI (ctypes on libpagedattn.so) and
compares its output with pa_decode's on the same inputs, within the parity
tolerance, on two calls in a row with different inputs (the shared scratch
keeps the first call's contents when the second runs), and both with the fp64
oracle.  This file is collected
last so that a stop-at-first-failure run has executed every other test first.
"""
import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_325_b200 as pa
from paged_kv_cache_325_b200 import workloads as W
from gpu_helpers import MAX_ABS, MEAN_ABS, DecodeOnGpu, assert_close, oracle_decode

pytestmark = pytest.mark.gpu

P = ctypes.c_void_p


def _noalloc(lib, g, out):
    c = g.case
    stream = torch.cuda.current_stream(g.dev).cuda_stream
    return lib.pa_decode_noalloc(P(out.data_ptr()), P(g.q.data_ptr()), P(g.k_cache.data_ptr()),
                                 P(g.v_cache.data_ptr()), P(g.block_table.data_ptr()), g.block_table.shape[1],
                                 P(g.context_lens.data_ptr()), c.batch, c.max_context_len, c.num_q_heads,
                                 c.num_kv_heads, c.head_dim, c.num_blocks, c.block_size, c.softmax_scale, None,
                                 P(stream))


def test_noalloc_matches_pa_decode_on_two_calls_in_a_row(cuda_lib):
    lib = pa.load_library()
    cases = [W.make_decode_case([3000, 777, 4100, 64, 2500], 32, 8, 128, 256, seed=1201),   # split path
             W.make_decode_case([1, 17, 100, 255, 900], 8, 2, 64, 16, seed=1202)]           # other shapes
    for case in cases:
        need = pa.pa_decode_workspace_size(case.batch, case.num_q_heads, case.num_kv_heads, case.head_dim,
                                           case.max_context_len, case.block_size)
        assert need <= lib.pa_decode_noalloc_max_scratch_bytes()
    assert pa.pa_decode_workspace_size(5, 32, 8, 128, 4100, 256) > 0   # the first case uses the scratch
    for case in cases:
        g = DecodeOnGpu(case)
        g.store()
        ref = g.decode()                                   # existing entry point, caller workspace
        got = torch.full_like(g.q, float("nan"))
        st = _noalloc(lib, g, got)
        assert st == pa.PA_OK, lib.pa_last_error_detail().decode()
        torch.cuda.synchronize()
        a = got.float().cpu().numpy()
        b = ref.float().cpu().numpy()
        assert np.isfinite(a).all()
        err = np.abs(a - b)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (case.name, err.max(), err.mean())
        assert_close(got, oracle_decode(case), what=f"noalloc {case.name} vs oracle")


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_lib):
    lib = pa.load_library()
    cap = lib.pa_decode_noalloc_max_scratch_bytes()
    batch, Hq, Hkv, D, ctx, B = 256, 32, 8, 128, 65536, 256
    assert pa.pa_decode_workspace_size(batch, Hq, Hkv, D, ctx, B) > cap
    st = lib.pa_decode_noalloc(None, None, None, None, None, 256, None, batch, ctx, Hq, Hkv, D, 70000, B, 0.088,
                               None, None)
    assert st == pa.PA_ERR_WORKSPACE
    assert "fixed array" in lib.pa_last_error_detail().decode()
