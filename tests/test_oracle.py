"""Pins for the CPU oracle: every check compares it with something other than itself.

* closed forms derived by hand from the pages' definitions (tests/golden);
* brute force in pure Python (math.fsum) on the generator's contiguous
  per-sequence source, so the oracle's paged gather is checked against data
  that never went through a block table;
* invariants of softmax attention (context 1, identical keys, key shift,
  dominant key, key order, block relabelling);
* a library cross-check against torch's fp64 scaled_dot_product_attention;
* prefill rows against decode with the matching context;
* planted mistakes (mutants of pa_oracle.c compiled on the CPU) must each
  fail at least one of these pins.
"""
import json
import math
import os
import tempfile

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_325_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_form.json")


def bf16(x) -> torch.Tensor:
    t = torch.tensor(x, dtype=torch.float64)
    b = t.to(torch.bfloat16)
    assert torch.equal(b.to(torch.float64), t), "fixture value is not bf16-exact"
    return b


def as_f(t: torch.Tensor):
    return t.to(torch.float64).tolist()


def brute_attend(q, K, V, scale):
    """softmax(scale * q.K_j) weighted sum of V_j with exactly rounded sums."""
    s = [scale * math.fsum(a * b for a, b in zip(q, k)) for k in K]
    m = max(s)
    w = [math.exp(x - m) for x in s]
    z = math.fsum(w)
    return [math.fsum(wj * v[d] for wj, v in zip(w, V)) / z for d in range(len(V[0]))]


# --------------------------------------------------------------------------
# individual pins; each takes an Oracle instance and raises AssertionError
# --------------------------------------------------------------------------

def _golden_cache(c):
    nb, B, Hkv, D = c["num_blocks"], c["B"], c["Hkv"], c["D"]
    k = np.zeros((nb * B, Hkv, D))
    v = np.zeros((nb * B, Hkv, D))
    for slot, rows in c["k_rows"].items():
        k[int(slot)] = rows
    for slot, rows in c["v_rows"].items():
        v[int(slot)] = rows
    return bf16(k.reshape(nb, B, Hkv, D)), bf16(v.reshape(nb, B, Hkv, D))


def pin_golden(orc):
    cases = json.load(open(GOLDEN))["cases"]
    for c in cases:
        kc, vc = _golden_cache(c)
        q = bf16(c["q"])
        if c["kind"] == "decode":
            out = orc.decode(q, kc, vc, c["block_table"], c["context_lens"], c["scale"])
        else:
            out = orc.prefill(q, kc, vc, c["cu_seqlens_q"], c["cu_seqlens_k"], c["block_table"], c["scale"],
                              causal=c["causal"])
        exp = np.array(c["expected"], dtype=np.float64)
        assert np.allclose(out, exp, rtol=0, atol=1e-12), (c["name"], out, exp)


def _tiny_decode_cases():
    yield W.make_decode_case([1, 2, 3], 2, 1, 8, 1, seed=11)
    yield W.make_decode_case([1, 3, 4, 6], 4, 2, 8, 2, seed=12)
    yield W.make_decode_case([5, 16, 17, 40], 4, 2, 8, 16, seed=13)
    yield W.make_decode_case([33, 20], 6, 3, 4, 16, seed=14)
    yield W.make_decode_case([19, 25], 4, 1, 8, 8, seed=15, shared_prefix_blocks=2)


def _post_store(orc, case):
    return orc.store(case.k_new, case.v_new, case.slot_mapping, case.k_cache, case.v_cache)


def pin_bruteforce_decode(orc):
    for case in _tiny_decode_cases():
        kc, vc = _post_store(orc, case)
        out = orc.decode(case.q, kc, vc, case.block_table, case.context_lens, case.softmax_scale)
        G = case.num_q_heads // case.num_kv_heads
        for s in range(case.batch):
            K = case.k_seq[s].to(torch.float64)
            V = case.v_seq[s].to(torch.float64)
            for h in range(case.num_q_heads):
                ref = brute_attend(as_f(case.q[s, h]), K[:, h // G].tolist(), V[:, h // G].tolist(),
                                   case.softmax_scale)
                assert np.allclose(out[s, h], ref, rtol=0, atol=1e-12), (case.name, s, h)


def _tiny_prefill_cases():
    yield W.make_prefill_case([5, 9, 1], [0, 4, 0], 4, 2, 8, 4, seed=21)
    yield W.make_prefill_case([17, 33, 16], [16, 16, 0], 2, 2, 8, 16, seed=22)
    yield W.make_prefill_case([3, 7], [2, 0], 3, 1, 4, 1, seed=23)


def pin_bruteforce_prefill(orc):
    for case in _tiny_prefill_cases():
        kc, vc = _post_store(orc, case)
        out = orc.prefill(case.q, kc, vc, case.cu_seqlens_q, case.cu_seqlens_k, case.block_table,
                          case.softmax_scale, causal=True)
        G = case.num_q_heads // case.num_kv_heads
        for s in range(case.batch):
            c = int(case.cached_lens[s])
            K = case.k_seq[s].to(torch.float64)
            V = case.v_seq[s].to(torch.float64)
            for i in range(int(case.cu_seqlens_q[s + 1] - case.cu_seqlens_q[s])):
                t = int(case.cu_seqlens_q[s]) + i
                for h in range(case.num_q_heads):
                    n = c + i + 1
                    ref = brute_attend(as_f(case.q[t, h]), K[:n, h // G].tolist(), V[:n, h // G].tolist(),
                                       case.softmax_scale)
                    assert np.allclose(out[t, h], ref, rtol=0, atol=1e-12), (case.name, s, i, h)


def _relabel(case, kc, vc, seed):
    """Move every physical block to a new random id: same sequences, other layout."""
    nb = kc.shape[0]
    pi = np.random.default_rng(seed).permutation(nb).astype(np.int32)
    kc2 = torch.empty_like(kc)
    vc2 = torch.empty_like(vc)
    kc2[torch.from_numpy(pi).long()] = kc
    vc2[torch.from_numpy(pi).long()] = vc
    bt = case.block_table.copy()
    bt[bt >= 0] = pi[bt[bt >= 0]]
    return kc2, vc2, bt


def pin_block_permutation(orc):
    case = W.make_decode_case([7, 30, 64, 3], 4, 2, 8, 4, seed=31)
    kc, vc = _post_store(orc, case)
    base = orc.decode(case.q, kc, vc, case.block_table, case.context_lens, case.softmax_scale)
    for seed in (1, 2):
        kc2, vc2, bt2 = _relabel(case, kc, vc, seed)
        out = orc.decode(case.q, kc2, vc2, bt2, case.context_lens, case.softmax_scale)
        assert np.array_equal(out, base), "paged result depends on the physical block ids"


def pin_context_one(orc):
    case = W.make_decode_case([1, 1, 1], 4, 2, 16, 16, seed=41)
    kc, vc = _post_store(orc, case)
    out = orc.decode(case.q, kc, vc, case.block_table, case.context_lens, case.softmax_scale)
    for s in range(3):
        for h in range(4):
            assert np.array_equal(out[s, h], case.v_new[s, h // 2].to(torch.float64).numpy())


def pin_identical_keys(orc):
    case = W.make_decode_case([9, 40], 2, 1, 8, 8, seed=51)
    kc, vc = _post_store(orc, case)
    row = case.k_new[0, 0].clone()
    kc[:] = row                        # every key in the cache is the same vector
    out = orc.decode(case.q, kc, vc, case.block_table, case.context_lens, case.softmax_scale)
    for s in range(2):
        mean = case.v_seq[s][:, 0].to(torch.float64).mean(0).numpy()
        for h in range(2):
            assert np.allclose(out[s, h], mean, rtol=0, atol=1e-12)


def _grid_values(rng, shape, lo=-16, hi=16):
    return torch.from_numpy(rng.integers(lo, hi + 1, size=shape) / 8.0).to(torch.bfloat16)


def pin_shift_invariance(orc):
    rng = np.random.default_rng(61)
    nb, B, Hkv, D = 4, 4, 1, 8
    kc = _grid_values(rng, (nb, B, Hkv, D))
    vc = _grid_values(rng, (nb, B, Hkv, D))
    q = _grid_values(rng, (2, 2, D))
    bt = np.array([[2, 0, 3], [1, 3, -1]], dtype=np.int32)
    ctx = np.array([11, 6], dtype=np.int32)
    u = _grid_values(rng, (D,))
    kc_shift = (kc.to(torch.float64) + u.to(torch.float64)).to(torch.bfloat16)
    assert torch.equal(kc_shift.to(torch.float64), kc.to(torch.float64) + u.to(torch.float64))
    a = orc.decode(q, kc, vc, bt, ctx, 0.3)
    b = orc.decode(q, kc_shift, vc, bt, ctx, 0.3)
    assert np.allclose(a, b, rtol=0, atol=1e-12), "adding one vector to every key changed the output"


def pin_dominant_key(orc):
    case = W.make_decode_case([50], 1, 1, 16, 16, seed=71)
    kc, vc = _post_store(orc, case)
    q = case.q[0, 0].to(torch.float64)
    j_star = 23
    kstar = (q * 8.0).to(torch.bfloat16)
    blk = int(case.block_table[0, j_star // 16])
    kc[blk, j_star % 16, 0] = kstar
    scale = case.softmax_scale
    scores = []
    for j in range(50):
        b = int(case.block_table[0, j // 16])
        scores.append(scale * float(q @ kc[b, j % 16, 0].to(torch.float64)))
    gap = scores[j_star] - max(s for j, s in enumerate(scores) if j != j_star)
    assert gap > 20
    out = orc.decode(case.q, kc, vc, case.block_table, case.context_lens, scale)
    vstar = vc[blk, j_star % 16, 0].to(torch.float64).numpy()
    vmax = float(case.v_seq[0].to(torch.float64).abs().max())
    bound = 49 * math.exp(-gap) * 2 * vmax + 1e-12
    assert np.abs(out[0, 0] - vstar).max() <= bound


def pin_key_order_invariance(orc):
    case = W.make_decode_case([13, 7], 2, 1, 8, 1, seed=81)  # block size 1: block order == key order
    kc, vc = _post_store(orc, case)
    a = orc.decode(case.q, kc, vc, case.block_table, case.context_lens, case.softmax_scale)
    bt = case.block_table.copy()
    rng = np.random.default_rng(3)
    for s in range(2):
        n = int(case.context_lens[s])
        bt[s, :n] = bt[s, rng.permutation(n)]
    b = orc.decode(case.q, kc, vc, bt, case.context_lens, case.softmax_scale)
    assert np.allclose(a, b, rtol=0, atol=1e-12)


def pin_prefill_equals_decode(orc):
    case = W.make_prefill_case([40, 23], [32, 0], 4, 2, 8, 8, seed=91)
    kc, vc = _post_store(orc, case)
    pre = orc.prefill(case.q, kc, vc, case.cu_seqlens_q, case.cu_seqlens_k, case.block_table,
                      case.softmax_scale, causal=True)
    full = orc.prefill(case.q, kc, vc, case.cu_seqlens_q, case.cu_seqlens_k, case.block_table,
                       case.softmax_scale, causal=False)
    for s in range(case.batch):
        c = int(case.cached_lens[s])
        n_k = int(case.prompt_lens[s])
        for i in range(n_k - c):
            t = int(case.cu_seqlens_q[s]) + i
            q1 = case.q[t:t + 1]
            dec = orc.decode(q1, kc, vc, case.block_table[s:s + 1], [c + i + 1], case.softmax_scale)
            assert np.array_equal(pre[t], dec[0]), (s, i)
            dec_all = orc.decode(q1, kc, vc, case.block_table[s:s + 1], [n_k], case.softmax_scale)
            assert np.array_equal(full[t], dec_all[0]), (s, i)


def pin_sdpa_crosscheck(orc):
    F = torch.nn.functional
    case = W.make_prefill_case([37, 64, 5], [16, 32, 0], 8, 2, 16, 16, seed=101)
    kc, vc = _post_store(orc, case)
    out = orc.prefill(case.q, kc, vc, case.cu_seqlens_q, case.cu_seqlens_k, case.block_table,
                      case.softmax_scale, causal=True)
    G = case.num_q_heads // case.num_kv_heads
    for s in range(case.batch):
        a, b = int(case.cu_seqlens_q[s]), int(case.cu_seqlens_q[s + 1])
        n_k = int(case.prompt_lens[s])
        c = n_k - (b - a)
        q = case.q[a:b].to(torch.float64).transpose(0, 1).unsqueeze(0)               # [1, Hq, n, D]
        K = case.k_seq[s].to(torch.float64).repeat_interleave(G, dim=1).transpose(0, 1).unsqueeze(0)
        V = case.v_seq[s].to(torch.float64).repeat_interleave(G, dim=1).transpose(0, 1).unsqueeze(0)
        qi = torch.arange(b - a).unsqueeze(1)
        kj = torch.arange(n_k).unsqueeze(0)
        mask = kj <= (c + qi)                                                        # bottom-right causal
        ref = F.scaled_dot_product_attention(q, K, V, attn_mask=mask, scale=case.softmax_scale)
        ref = ref[0].transpose(0, 1).numpy()
        assert np.allclose(out[a:b], ref, rtol=0, atol=1e-10), s


def pin_store(orc):
    rng = np.random.default_rng(111)
    nb, B, Hkv, D = 6, 4, 2, 8
    kc = torch.from_numpy(rng.standard_normal((nb, B, Hkv, D)).astype(np.float32)).to(torch.bfloat16)
    vc = torch.from_numpy(rng.standard_normal((nb, B, Hkv, D)).astype(np.float32)).to(torch.bfloat16)
    N = 9
    k = torch.from_numpy(rng.standard_normal((N, Hkv, D)).astype(np.float32)).to(torch.bfloat16)
    v = torch.from_numpy(rng.standard_normal((N, Hkv, D)).astype(np.float32)).to(torch.bfloat16)
    slots = rng.permutation(nb * B)[:N].astype(np.int32)
    slots[[2, 5]] = -1
    k2, v2 = orc.store(k, v, slots, kc, vc)
    ek = kc.reshape(nb * B, Hkv, D).clone()
    ev = vc.reshape(nb * B, Hkv, D).clone()
    for i, s in enumerate(slots):
        if s >= 0:
            ek[s] = k[i]
            ev[s] = v[i]
    assert torch.equal(k2.reshape(-1).view(torch.int16), ek.reshape(-1).view(torch.int16))
    assert torch.equal(v2.reshape(-1).view(torch.int16), ev.reshape(-1).view(torch.int16))
    with pytest.raises(ValueError):
        orc.store(k[:1], v[:1], [nb * B], kc, vc)


PINS = [pin_golden, pin_bruteforce_decode, pin_bruteforce_prefill, pin_block_permutation, pin_context_one,
        pin_identical_keys, pin_shift_invariance, pin_dominant_key, pin_key_order_invariance,
        pin_prefill_equals_decode, pin_sdpa_crosscheck, pin_store]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(oracle.default())


# --------------------------------------------------------------------------
# planted mistakes: each mutant of the oracle source must fail some pin
# --------------------------------------------------------------------------

# Every mutant keeps its memory accesses inside the buffers (it runs in this process).
MUTANTS = {
    "slot_block_not_scaled": ("bt_row[p / block_size] * block_size + p % block_size",
                              "bt_row[p / block_size] + p % block_size"),
    "gqa_interleaved": ("int32_t kvh = h / group;", "int32_t kvh = h % num_kv_heads;"),
    "scale_dropped": ("score[j] = scale * dot;", "score[j] = dot;"),
    "causal_ignores_cached_prefix": ("causal ? c + i + 1 : n_k", "causal ? i + 1 : n_k"),
    "causal_off_by_one": ("causal ? c + i + 1 : n_k", "causal ? c + i : n_k"),
    "max_sign_flipped": ("score[j] = exp(score[j] - m);", "score[j] = exp(m - score[j]);"),
    "normaliser_dropped": ("out[d] = acc / z;", "out[d] = acc;"),
    "v_from_k_in_store": ("memcpy(v_cache + slot * row, v +", "memcpy(v_cache + slot * row, k +"),
    "gather_wrong_head": ("(slot * num_kv_heads + kv_head)", "(slot * num_kv_heads + 0)"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "pa_oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, f"mutation anchor missing: {old}"
    with tempfile.TemporaryDirectory() as d:
        path = os.path.join(d, "mutant.c")
        open(path, "w").write(src.replace(old, new))
        mutant = oracle.Oracle(oracle.compile_oracle(path, os.path.join(d, "libmutant.so")))
        failed = []
        for pin in PINS:
            try:
                pin(mutant)
            except (AssertionError, ValueError):
                failed.append(pin.__name__)
        assert failed, f"mutant {name} passed every pin"
