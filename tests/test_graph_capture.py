"""Fixed-shape store + decode captured once in a CUDA graph and replayed.

The small-batch decode the pages speed up with graph replay (nano-vllm
walkthrough: CUDA graphs captured at start-up, then replayed) runs here on
static buffers: a padded batch whose padding rows carry slot_mapping = -1 (the
store skips them) and a one-token context on a spare block.  Each replay takes
new inputs copied into the static buffers; the real rows are checked against
the oracle every step.  Both forms are captured: pa_store_kv then pa_decode,
and pa_store_kv_decode (the store inside the decode launch).
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_325_b200 as pa
from paged_kv_cache_325_b200 import workloads as W
from gpu_helpers import assert_close

pytestmark = pytest.mark.gpu


def _step_case(step, n_real, pad, Hq, Hkv, D, B):
    """A decode step of n_real sequences plus `pad` padding rows, as host arrays."""
    rng = np.random.default_rng(50 + step)
    ctx = rng.integers(20, 700, size=n_real)
    case = W.make_decode_case(ctx, Hq, Hkv, D, B, seed=1500 + step, num_blocks=64 * 8)
    used = set(case.block_table[case.block_table >= 0].tolist())
    spare = min(set(range(case.num_blocks)) - used)  # a block no real sequence uses
    bt = np.full((n_real + pad, case.block_table.shape[1]), -1, dtype=np.int32)
    bt[:n_real] = case.block_table
    bt[n_real:, 0] = spare
    ctx_all = np.concatenate([case.context_lens, np.ones(pad, dtype=np.int32)])
    slots = np.concatenate([case.slot_mapping, -np.ones(pad, dtype=np.int32)])
    q = torch.cat([case.q, torch.zeros(pad, Hq, D, dtype=torch.bfloat16)])
    kn = torch.cat([case.k_new, torch.zeros(pad, Hkv, D, dtype=torch.bfloat16)])
    vn = torch.cat([case.v_new, torch.zeros(pad, Hkv, D, dtype=torch.bfloat16)])
    case.k_cache[spare] = 0                          # the padding rows read a finite block
    case.v_cache[spare] = 0
    return case, bt, ctx_all, slots, q, kn, vn


@pytest.mark.parametrize("fused", [False, True], ids=["store_then_decode", "pa_store_kv_decode"])
def test_store_and_decode_replay_from_a_cuda_graph(cuda_lib, fused):
    dev = torch.device("cuda:0")
    n_real, pad, Hq, Hkv, D, B, maxb = 13, 3, 16, 8, 128, 16, 48
    batch = n_real + pad
    max_ctx = maxb * B
    # static buffers, sized once
    case0 = _step_case(0, n_real, pad, Hq, Hkv, D, B)[0]
    kc = torch.empty_like(case0.k_cache, device=dev)
    vc = torch.empty_like(case0.v_cache, device=dev)
    q = torch.empty(batch, Hq, D, dtype=torch.bfloat16, device=dev)
    kn = torch.empty(batch, Hkv, D, dtype=torch.bfloat16, device=dev)
    vn = torch.empty_like(kn)
    slots = torch.empty(batch, dtype=torch.int32, device=dev)
    bt = torch.full((batch, maxb), -1, dtype=torch.int32, device=dev)
    ctx = torch.empty(batch, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    ws = pa.alloc_decode_workspace(q, Hkv, max_ctx, B)

    def step():
        if fused:                            # one launch
            pa.pa_store_kv_decode(kn, vn, slots, out, q, kc, vc, bt, ctx, max_ctx, case0.softmax_scale, workspace=ws)
        else:
            pa.pa_store_kv(kn, vn, slots, kc, vc)
            pa.pa_decode(out, q, kc, vc, bt, ctx, max_ctx, case0.softmax_scale, workspace=ws)

    def load(step_no):
        case, bt_h, ctx_h, sl_h, q_h, kn_h, vn_h = _step_case(step_no, n_real, pad, Hq, Hkv, D, B)
        kc.copy_(case.k_cache)
        vc.copy_(case.v_cache)
        q.copy_(q_h)
        kn.copy_(kn_h)
        vn.copy_(vn_h)
        slots.copy_(torch.from_numpy(sl_h))
        bt.fill_(-1)
        bt[:, :bt_h.shape[1]].copy_(torch.from_numpy(bt_h))
        ctx.copy_(torch.from_numpy(ctx_h))
        return case

    load(0)
    step()                                   # first calls outside capture (library set-up)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g):
            step()
    torch.cuda.synchronize()

    for step_no in (1, 2, 3):
        case = load(step_no)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        kc_ref, vc_ref = oracle.store(case.k_new, case.v_new, case.slot_mapping, case.k_cache, case.v_cache)
        ref = oracle.decode(case.q, kc_ref, vc_ref, case.block_table, case.context_lens, case.softmax_scale)
        assert_close(out[:n_real], ref, what=f"graph replay step {step_no}")
        # the store wrote exactly the real rows: the cache equals the oracle's post-store cache
        assert torch.equal(kc.cpu().view(torch.int16), kc_ref.view(torch.int16))
