"""pa_store_kv on the GPU: bit-exact against the oracle's store."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_325_b200 as pa
from paged_kv_cache_325_b200 import workloads as W
from gpu_helpers import DecodeOnGpu, PrefillOnGpu, i32

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.detach().contiguous().view(torch.int16).cpu()


def _check_store(case, g):
    g.store()
    torch.cuda.synchronize()
    kc, vc = oracle.store(case.k_new, case.v_new, case.slot_mapping, case.k_cache, case.v_cache)
    assert torch.equal(_bits(g.k_cache), _bits(kc)), "k_cache differs from the oracle's store"
    assert torch.equal(_bits(g.v_cache), _bits(vc)), "v_cache differs from the oracle's store"


@pytest.mark.parametrize("make", [W.tiny_decode, W.qwen3_06b_decode], ids=["tiny", "qwen3_0.6b"])
def test_store_decode_workloads(cuda_lib, make):
    case = make()
    _check_store(case, DecodeOnGpu(case))


def test_store_varlen_prefill_workload(cuda_lib):
    case = W.varlen_prefill()
    _check_store(case, PrefillOnGpu(case))


@pytest.mark.parametrize("Hkv,D,B", [(1, 64, 16), (2, 128, 32), (8, 128, 256), (3, 64, 64)])
def test_store_shapes_and_padding_rows(cuda_lib, Hkv, D, B):
    case = W.make_decode_case(list(range(1, 40, 3)), Hkv * 2, Hkv, D, B, seed=7 + Hkv)
    case.slot_mapping[[1, 4]] = -1               # padding rows: must not be written
    _check_store(case, DecodeOnGpu(case))


def test_store_strided_rows_from_a_fused_qkv_buffer(cuda_lib):
    dev = torch.device("cuda:0")
    N, Hq, Hkv, D, B, nb = 37, 16, 8, 128, 16, 8
    qkv = torch.randn(N, (Hq + 2 * Hkv) * D, device=dev).to(torch.bfloat16)
    k = qkv[:, Hq * D:(Hq + Hkv) * D].view(N, Hkv, D)
    v = qkv[:, (Hq + Hkv) * D:].view(N, Hkv, D)
    slots = torch.randperm(nb * B, device=dev)[:N].to(torch.int32)
    kc = torch.zeros(nb, B, Hkv, D, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    pa.pa_store_kv(k, v, slots, kc, vc)
    ek = torch.zeros_like(kc).view(-1, Hkv, D)
    ev = torch.zeros_like(vc).view(-1, Hkv, D)
    ek[slots.long()] = k
    ev[slots.long()] = v
    torch.cuda.synchronize()
    assert torch.equal(_bits(kc.view(-1, Hkv, D)), _bits(ek))
    assert torch.equal(_bits(vc.view(-1, Hkv, D)), _bits(ev))


def test_store_unaligned_row_stride_takes_the_scalar_path(cuda_lib):
    dev = torch.device("cuda:0")
    N, Hkv, D, B, nb = 9, 2, 64, 16, 4
    buf = torch.randn(N, Hkv * D + 3, device=dev).to(torch.bfloat16)   # row stride 131 elements
    k = buf[:, :Hkv * D].view(N, Hkv, D)
    v = buf[:, 3:3 + Hkv * D].view(N, Hkv, D)
    slots = torch.arange(N, device=dev, dtype=torch.int32) * 3
    kc = torch.zeros(nb, B, Hkv, D, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    pa.pa_store_kv(k, v, slots, kc, vc)
    torch.cuda.synchronize()
    assert torch.equal(_bits(kc.view(-1, Hkv, D)[slots.long()]), _bits(k))
    assert torch.equal(_bits(vc.view(-1, Hkv, D)[slots.long()]), _bits(v))


def test_store_checked_mode_flags_slots_past_the_cache(cuda_lib):
    dev = torch.device("cuda:0")
    N, Hkv, D, B, nb = 4, 2, 64, 16, 2
    k = torch.randn(N, Hkv, D, device=dev).to(torch.bfloat16)
    slots = i32([0, nb * B, 5, -1], dev)       # slot 32 is one past the end
    kc = torch.zeros(nb, B, Hkv, D, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    pa.pa_store_kv(k, k, slots, kc, vc, dev_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & pa.PA_DEVERR_SLOT
    flat = kc.view(-1, Hkv, D)
    assert torch.equal(_bits(flat[0]), _bits(k[0])) and torch.equal(_bits(flat[5]), _bits(k[2]))
    assert int((flat.float() != 0).any(-1).any(-1).sum()) == 2


def test_store_empty_is_a_noop(cuda_lib):
    dev = torch.device("cuda:0")
    kc = torch.zeros(2, 16, 1, 64, dtype=torch.bfloat16, device=dev)
    e = torch.empty(0, 1, 64, dtype=torch.bfloat16, device=dev)
    pa.pa_store_kv(e, e, torch.empty(0, dtype=torch.int32, device=dev), kc, kc)
    torch.cuda.synchronize()
    assert not kc.float().any()
