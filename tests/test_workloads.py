"""The seeded input generator: determinism and the structure of each workload."""
import numpy as np
import torch

from paged_kv_cache_325_b200 import workloads as W


def _bits(t):
    return t.contiguous().view(torch.int16)


def test_deterministic():
    a = W.tiny_decode()
    b = W.tiny_decode()
    assert torch.equal(_bits(a.k_cache), _bits(b.k_cache))
    assert torch.equal(_bits(a.q), _bits(b.q))
    assert np.array_equal(a.block_table, b.block_table)


def test_tiny_decode_structure():
    c = W.tiny_decode()
    assert c.batch == 4 and list(c.context_lens) == [1, 17, 100, 255]
    assert c.num_blocks == 64 and c.block_size == 16
    used = c.block_table[c.block_table >= 0]
    assert len(used) == 1 + 2 + 7 + 16 and len(set(used.tolist())) == len(used)
    assert used.max() < 64


def test_poison_marks_uncovered_slots():
    c = W.make_decode_case([5, 20], 2, 1, 8, 4, seed=3, num_blocks=12)
    nan = torch.isnan(c.k_cache.float()).all(-1).all(-1)   # [nb, B]
    for s, n in enumerate(c.context_lens):
        for p in range(int(n) - 1):                         # history is finite
            blk = c.block_table[s, p // 4]
            assert not nan[blk, p % 4]
        blk = c.block_table[s, (n - 1) // 4]                # the slot the store fills is poisoned
        assert nan[blk, (n - 1) % 4]
    assert int(nan.sum()) == 12 * 4 - (4 + 19)


def test_slot_mapping_points_at_the_newest_position():
    c = W.make_decode_case([3, 9, 16], 2, 2, 8, 4, seed=4)
    for s, n in enumerate(c.context_lens):
        blk, off = divmod(int(c.slot_mapping[s]), 4)
        assert blk == c.block_table[s, (n - 1) // 4] and off == (n - 1) % 4


def test_prefix_sharing_structure():
    c = W.make_decode_case([4097, 4200, 4500], 2, 1, 8, 256, seed=5, shared_prefix_blocks=16,
                           keep_contiguous=False)
    assert (c.block_table[:, :16] == c.block_table[0, :16]).all()
    private = c.block_table[:, 16:][c.block_table[:, 16:] >= 0]
    assert len(set(private.tolist())) == len(private)
    assert not set(private.tolist()) & set(c.block_table[0, :16].tolist())


def test_varlen_prefill_structure():
    c = W.varlen_prefill()
    assert c.batch == 12 and c.block_size == 256
    assert ((c.prompt_lens >= 128) & (c.prompt_lens <= 2048)).all()
    assert (c.cached_lens % 256 == 0).all() and (c.cached_lens[1::2] == 0).all()
    assert (c.prompt_lens - c.cached_lens >= 1).all()
    assert np.array_equal(np.diff(c.cu_seqlens_k), c.prompt_lens)
    assert np.array_equal(np.diff(c.cu_seqlens_q), c.prompt_lens - c.cached_lens)
    assert c.q.shape == (c.total_q, 32, 128) and c.k_new.shape == (c.total_q, 8, 128)
