"""The C-ABI library on the CPU: it loads, exports every declared entry point,
and rejects bad host-side arguments before touching CUDA.

Every call here fails validation before any CUDA call is made, so these tests
are safe with or without a GPU (fake pointers are never dereferenced).
"""
import ctypes
import subprocess

import pytest

import paged_kv_cache_325_b200 as pa
from paged_kv_cache_325_b200 import _binding

P = ctypes.c_void_p
A = P(0x10000)          # an aligned fake device address (never dereferenced)
MIS = P(0x10002)        # misaligned


@pytest.fixture(scope="module")
def lib():
    return pa.load_library()


def test_exports_every_declared_symbol(lib):
    declared = pa.declared_symbols()
    assert {"pa_store_kv", "pa_decode", "pa_prefill_varlen"} <= set(declared)
    out = subprocess.run(["nm", "-D", "--defined-only", _binding.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [s for s in declared if s not in exported]
    assert not missing, missing
    for s in declared:
        assert hasattr(lib, s)


def test_status_strings(lib):
    assert pa.pa_status_string(0) == "PA_OK"
    assert pa.pa_status_string(6) == "PA_ERR_WORKSPACE"
    assert pa.pa_status_string(99) == "PA_ERR_UNKNOWN"
    assert pa.pa_version() >= 100


def _store(lib, **kw):
    a = dict(k=A, v=A, ks=2048, vs=2048, slots=A, n=4, kc=A, vc=A, nb=8, B=256, Hkv=8, D=128, err=None)
    a.update(kw)
    return lib.pa_store_kv(a["k"], a["v"], a["ks"], a["vs"], a["slots"], a["n"], a["kc"], a["vc"], a["nb"],
                           a["B"], a["Hkv"], a["D"], a["err"], None)


def test_store_validation(lib):
    assert _store(lib, D=96) == pa.PA_ERR_UNSUPPORTED
    assert _store(lib, B=24) == pa.PA_ERR_UNSUPPORTED
    assert _store(lib, B=512) == pa.PA_ERR_UNSUPPORTED
    assert _store(lib, n=-1) == pa.PA_ERR_INVALID_ARG
    assert _store(lib, ks=100) == pa.PA_ERR_INVALID_ARG
    assert _store(lib, k=None) == pa.PA_ERR_INVALID_ARG
    assert _store(lib, kc=MIS) == pa.PA_ERR_INVALID_ARG
    assert _store(lib, nb=0) == pa.PA_ERR_INVALID_ARG
    assert _store(lib, nb=1 << 24, B=256) == pa.PA_ERR_UNSUPPORTED
    assert "num_blocks" in lib.pa_last_error_detail().decode()
    assert _store(lib, n=0, k=None, v=None) == pa.PA_OK          # empty store is a no-op


def _decode(lib, **kw):
    a = dict(out=A, q=A, kc=A, vc=A, bt=A, bts=4, ctx=A, batch=2, maxc=1000, Hq=32, Hkv=8, D=128, nb=16, B=256,
             scale=0.088, ws=None, wsb=0, err=None)
    a.update(kw)
    return lib.pa_decode(a["out"], a["q"], a["kc"], a["vc"], a["bt"], a["bts"], a["ctx"], a["batch"], a["maxc"],
                         a["Hq"], a["Hkv"], a["D"], a["nb"], a["B"], a["scale"], a["ws"], a["wsb"], a["err"], None)


def test_decode_validation(lib):
    assert _decode(lib, Hq=30) == pa.PA_ERR_INVALID_ARG
    assert _decode(lib, Hq=64, Hkv=2) == pa.PA_ERR_UNSUPPORTED      # group 32
    assert _decode(lib, D=256) == pa.PA_ERR_UNSUPPORTED
    assert _decode(lib, scale=0.0) == pa.PA_ERR_INVALID_ARG
    assert _decode(lib, scale=float("nan")) == pa.PA_ERR_INVALID_ARG
    assert _decode(lib, maxc=0) == pa.PA_ERR_INVALID_ARG
    assert _decode(lib, bts=0) == pa.PA_ERR_INVALID_ARG
    assert _decode(lib, q=None) == pa.PA_ERR_INVALID_ARG
    assert _decode(lib, out=MIS) == pa.PA_ERR_INVALID_ARG
    assert _decode(lib, batch=0) == pa.PA_OK
    # a long context needs a split workspace; none given
    assert _decode(lib, maxc=32768, batch=8) == pa.PA_ERR_WORKSPACE
    assert _decode(lib, maxc=32768, batch=8, ws=A, wsb=16) == pa.PA_ERR_WORKSPACE


def _store_decode(lib, **kw):
    a = dict(k=A, v=A, ks=1024, vs=1024, slots=A, out=A, q=A, kc=A, vc=A, bt=A, bts=4, ctx=A, batch=2, maxc=1000,
             Hq=32, Hkv=8, D=128, nb=16, B=256, scale=0.088, ws=None, wsb=0, err=None)
    a.update(kw)
    return lib.pa_store_kv_decode(a["k"], a["v"], a["ks"], a["vs"], a["slots"], a["out"], a["q"], a["kc"], a["vc"],
                                  a["bt"], a["bts"], a["ctx"], a["batch"], a["maxc"], a["Hq"], a["Hkv"], a["D"],
                                  a["nb"], a["B"], a["scale"], a["ws"], a["wsb"], a["err"], None)


def test_store_decode_validation(lib):
    assert _store_decode(lib, k=None) == pa.PA_ERR_INVALID_ARG
    assert _store_decode(lib, slots=None) == pa.PA_ERR_INVALID_ARG
    assert _store_decode(lib, ks=1000) == pa.PA_ERR_INVALID_ARG            # shorter than one row
    assert _store_decode(lib, ks=1028) == pa.PA_ERR_UNSUPPORTED            # rows not 16-byte aligned
    assert _store_decode(lib, v=MIS) == pa.PA_ERR_UNSUPPORTED
    assert "pa_store_kv then pa_decode" in lib.pa_last_error_detail().decode()
    assert _store_decode(lib, slots=MIS) == pa.PA_ERR_INVALID_ARG
    assert _store_decode(lib, D=96) == pa.PA_ERR_UNSUPPORTED
    assert _store_decode(lib, batch=0) == pa.PA_OK
    assert _store_decode(lib, maxc=32768, batch=8) == pa.PA_ERR_WORKSPACE


def _store_prefill(lib, **kw):
    a = dict(k=A, v=A, ks=1024, vs=1024, slots=A, out=A, q=A, tq=150, kc=A, vc=A, cq=A, ck=A, mq=100, mk=200, bt=A,
             bts=4, batch=2, Hq=32, Hkv=8, D=128, nb=16, B=256, scale=0.088, causal=1, ws=A, wsb=1 << 20, err=None)
    a.update(kw)
    return lib.pa_store_kv_prefill_varlen(a["k"], a["v"], a["ks"], a["vs"], a["slots"], a["out"], a["q"], a["tq"],
                                          a["kc"], a["vc"], a["cq"], a["ck"], a["mq"], a["mk"], a["bt"], a["bts"],
                                          a["batch"], a["Hq"], a["Hkv"], a["D"], a["nb"], a["B"], a["scale"],
                                          a["causal"], a["ws"], a["wsb"], a["err"], None)


def test_store_prefill_validation(lib):
    assert _store_prefill(lib, k=None) == pa.PA_ERR_INVALID_ARG
    assert _store_prefill(lib, slots=None) == pa.PA_ERR_INVALID_ARG
    assert _store_prefill(lib, vs=1000) == pa.PA_ERR_INVALID_ARG            # shorter than one row
    assert _store_prefill(lib, ks=1028) == pa.PA_ERR_UNSUPPORTED            # rows not 16-byte aligned
    assert _store_prefill(lib, k=MIS) == pa.PA_ERR_UNSUPPORTED
    assert "pa_store_kv then pa_prefill_varlen" in lib.pa_last_error_detail().decode()
    assert _store_prefill(lib, Hq=48, Hkv=8) == pa.PA_ERR_UNSUPPORTED        # group 6 does not divide 128
    assert _store_prefill(lib, tq=0) == pa.PA_OK                              # nothing to do
    assert _store_prefill(lib, ws=None, wsb=0) == pa.PA_ERR_WORKSPACE


def test_mixed_validation(lib):
    def call(**kw):
        a = dict(out=A, q=A, tq=150, kc=A, vc=A, cq=A, ck=A, mq=100, mk=2000, bt=A, bts=8, batch=4, Hq=32, Hkv=8,
                 D=128, nb=64, B=256, scale=0.088, ws=A, wsb=1 << 26, err=None)
        a.update(kw)
        return lib.pa_prefill_varlen_mixed(a["out"], a["q"], a["tq"], a["kc"], a["vc"], a["cq"], a["ck"], a["mq"],
                                           a["mk"], a["bt"], a["bts"], a["batch"], a["Hq"], a["Hkv"], a["D"], a["nb"],
                                           a["B"], a["scale"], a["ws"], a["wsb"], a["err"], None)
    assert call(ws=None, wsb=0) == pa.PA_ERR_WORKSPACE
    assert call(wsb=256) == pa.PA_ERR_WORKSPACE
    assert call(Hq=48) == pa.PA_ERR_UNSUPPORTED          # GQA group 6 does not divide 128
    assert call(Hq=30) == pa.PA_ERR_INVALID_ARG
    assert call(batch=0) == pa.PA_OK
    assert call(q=None) == pa.PA_ERR_INVALID_ARG
    n = pa.pa_prefill_varlen_mixed_workspace_size(4, 100, 2000, 32, 8, 128)
    assert n >= pa.pa_prefill_workspace_size(4, 100, 32, 8, 128) + pa.pa_decode_workspace_size(4, 32, 8, 128, 2000, 256)


def test_decode_workspace_size_query():
    assert pa.pa_decode_workspace_size(0, 32, 8, 128, 32768, 256) == 0
    n = pa.pa_decode_workspace_size(8, 32, 8, 128, 32768, 256)
    assert n > 0 and n % 4 == 0
    # explicit splits: 4 splits of a 1000-token context for 2 x 16 heads of 128
    n4 = pa.pa_decode_split_workspace_size(2, 16, 8, 128, 1000, 4)
    assert n4 >= 2 * 16 * 4 * (128 + 1) * 4
    n1 = pa.pa_decode_split_workspace_size(2, 16, 8, 128, 1000, 1)   # one split: the item table alone
    assert 0 < n1 < n4 and n1 % 256 == 0


def _prefill(lib, **kw):
    a = dict(out=A, q=A, tq=150, kc=A, vc=A, cq=A, ck=A, mq=100, mk=200, bt=A, bts=4, batch=2, Hq=32, Hkv=8, D=128,
             nb=16, B=256, scale=0.088, causal=1, err=None, ws=A, wsb=1 << 20)
    a.update(kw)
    return lib.pa_prefill_varlen(a["out"], a["q"], a["tq"], a["kc"], a["vc"], a["cq"], a["ck"], a["mq"], a["mk"],
                                 a["bt"], a["bts"], a["batch"], a["Hq"], a["Hkv"], a["D"], a["nb"], a["B"],
                                 a["scale"], a["causal"], a["ws"], a["wsb"], a["err"], None)


def test_prefill_validation(lib):
    assert _prefill(lib, Hq=12, Hkv=1) == pa.PA_ERR_UNSUPPORTED     # group 12 does not divide 128
    assert _prefill(lib, Hq=33) == pa.PA_ERR_INVALID_ARG
    assert _prefill(lib, mk=50) == pa.PA_ERR_INVALID_ARG            # max_seqlen_k < max_seqlen_q
    assert _prefill(lib, cq=None) == pa.PA_ERR_INVALID_ARG
    assert _prefill(lib, ck=P(0x10001)) == pa.PA_ERR_INVALID_ARG
    assert _prefill(lib, batch=0) == pa.PA_OK
    assert _prefill(lib, mq=0) == pa.PA_OK
    assert _prefill(lib, tq=0) == pa.PA_OK
    assert _prefill(lib, tq=-1) == pa.PA_ERR_INVALID_ARG
    assert _prefill(lib, ws=None, wsb=0) == pa.PA_ERR_WORKSPACE     # no workspace for the unit table
    need = pa.pa_prefill_workspace_size(2, 100, 32, 8, 128)
    assert need >= 4 * (16 + 2 + 1 + 2)
    assert _prefill(lib, ws=A, wsb=need - 1) == pa.PA_ERR_WORKSPACE
    assert _prefill(lib, batch=7000, ws=A, wsb=1 << 20) == pa.PA_ERR_UNSUPPORTED


def test_selftest_validation(lib):
    assert lib.pa_selftest_exp2(None, None, None, 4, None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_selftest_exp2(None, None, None, -1, None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_selftest_exp2(None, None, None, 0, None) == pa.PA_OK
    assert lib.pa_selftest_bounded_wait(None, 100, None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_selftest_bounded_wait(A, 0, None) == pa.PA_ERR_INVALID_ARG


def test_binding_rejects_cpu_tensors():
    import torch
    q = torch.zeros(2, 4, 64, dtype=torch.bfloat16)
    kc = torch.zeros(4, 16, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pa.pa_decode(q.clone(), q, kc, kc, torch.zeros(2, 1, dtype=torch.int32), torch.ones(2, dtype=torch.int32),
                     1, 0.125)


def test_binding_new_entry_points_reject_cpu_tensors():
    """No CPU path: every entry point refuses host tensors before calling the library."""
    import torch
    q = torch.zeros(2, 4, 64, dtype=torch.bfloat16)
    kv = torch.zeros(2, 2, 64, dtype=torch.bfloat16)
    kc = torch.zeros(4, 16, 2, 64, dtype=torch.bfloat16)
    i32 = lambda *shape: torch.zeros(*shape, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pa.pa_store_kv_decode(kv, kv, i32(2), q.clone(), q, kc, kc, i32(2, 1), i32(2), 16, 0.125)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pa.pa_store_kv_prefill_varlen(kv, kv, i32(2), q.clone(), q, kc, kc, i32(3), i32(3), 1, 1, i32(2, 1), 0.125)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pa.pa_prefill_varlen_mixed(q.clone(), q, kc, kc, i32(3), i32(3), 1, 1, i32(2, 1), 0.125)
