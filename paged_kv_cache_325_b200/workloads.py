"""Seeded synthetic inputs for the paged-KV hot path.

This module builds the bytes that both the CUDA path and the CPU oracle
consume. It holds no attention arithmetic: it draws random numbers, lays the
drawn tokens out in a block-paged cache the way a block manager and model
runner would (nano-vllm walkthrough, xingyun3d.csdn.net, section five
"KV Block 管理" and section seven "后端执行"), and records the host-side
metadata (block_table, slot_mapping, context_lens, cu_seqlens).

Recipe (all configurations):
  * generator: numpy ``Generator(PCG64(seed))``;
  * values: float32 N(0, 1) cast to bfloat16 with round-to-nearest-even;
  * physical blocks: ``rng.permutation(num_blocks)`` handed out in order of
    (sequence, logical block), so logically adjacent blocks are scattered;
  * ``num_blocks`` = blocks needed + 25 % slack unless a configuration fixes it;
  * ``poison=True`` fills every cache slot that no context covers, and the
    slots the store is about to write, with bf16 NaN, so a read outside a
    sequence's context (or a missing store) shows up as NaN in the output;
    ``poison=False`` fills them with N(0, 1) noise instead (timing runs).

The cache layout is ``[num_blocks, block_size, num_kv_heads, head_dim]``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np
import torch

BF16_NAN_BITS = 0x7FC0


def _normal_bf16(rng: np.random.Generator, shape) -> torch.Tensor:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    return torch.from_numpy(a).to(torch.bfloat16)


def _fill_bf16(shape, poison: bool, rng: np.random.Generator) -> torch.Tensor:
    if poison:
        t = torch.empty(shape, dtype=torch.bfloat16)
        t.view(torch.int16).fill_(BF16_NAN_BITS)
        return t
    return _normal_bf16(rng, shape)


def _with_slack(needed: int) -> int:
    return int(math.ceil(needed * 1.25))


@dataclass
class DecodeCase:
    """One decode step: store each sequence's newest K/V row, then attend."""

    name: str
    seed: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    context_lens: np.ndarray          # int32 [batch]; includes the token stored this step
    block_table: np.ndarray           # int32 [batch, max_blocks]; -1 past the last used block
    k_cache: torch.Tensor             # bf16 [nb, B, Hkv, D] before the store
    v_cache: torch.Tensor
    k_new: torch.Tensor               # bf16 [batch, Hkv, D]: K of token context_len-1
    v_new: torch.Tensor
    slot_mapping: np.ndarray          # int32 [batch]
    q: torch.Tensor                   # bf16 [batch, Hq, D]
    softmax_scale: float
    k_seq: Optional[List[torch.Tensor]] = None   # contiguous source [ctx, Hkv, D] per sequence
    v_seq: Optional[List[torch.Tensor]] = None
    shared_prefix_blocks: int = 0

    @property
    def batch(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.batch else 0

    def kv_bytes_read(self) -> int:
        """Logical K+V bytes one decode call reads (every sequence's context)."""
        row = self.num_kv_heads * self.head_dim * 2
        return int(self.context_lens.astype(np.int64).sum()) * row * 2

    def kv_bytes_unique(self) -> int:
        """K+V bytes of the distinct cache slots the contexts cover."""
        row = self.num_kv_heads * self.head_dim * 2
        slots = set()
        B = self.block_size
        for s in range(self.batch):
            n = int(self.context_lens[s])
            for i in range((n + B - 1) // B):
                used = min(B, n - i * B)
                slots.add((int(self.block_table[s, i]), used))
        per_block = {}
        for blk, used in slots:
            per_block[blk] = max(per_block.get(blk, 0), used)
        return sum(per_block.values()) * row * 2


@dataclass
class PrefillCase:
    """One varlen prefill step: store the new prompt tokens, then attend causally."""

    name: str
    seed: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    prompt_lens: np.ndarray           # int32 [batch]  (n_k per sequence)
    cached_lens: np.ndarray           # int32 [batch]  (whole blocks already in the cache)
    cu_seqlens_q: np.ndarray          # int32 [batch+1]
    cu_seqlens_k: np.ndarray          # int32 [batch+1]
    block_table: np.ndarray           # int32 [batch, max_blocks]
    k_cache: torch.Tensor             # bf16 [nb, B, Hkv, D] before the store
    v_cache: torch.Tensor
    k_new: torch.Tensor               # bf16 [total_q, Hkv, D]
    v_new: torch.Tensor
    slot_mapping: np.ndarray          # int32 [total_q]
    q: torch.Tensor                   # bf16 [total_q, Hq, D]
    softmax_scale: float
    causal: bool = True
    k_seq: Optional[List[torch.Tensor]] = None
    v_seq: Optional[List[torch.Tensor]] = None

    @property
    def batch(self) -> int:
        return int(self.prompt_lens.shape[0])

    @property
    def total_q(self) -> int:
        return int(self.cu_seqlens_q[-1])

    @property
    def max_seqlen_q(self) -> int:
        return int(np.diff(self.cu_seqlens_q).max()) if self.batch else 0

    @property
    def max_seqlen_k(self) -> int:
        return int(np.diff(self.cu_seqlens_k).max()) if self.batch else 0

    def causal_flops(self) -> int:
        """Multiply-add FLOPs of QK^T and PV over the causal pairs only."""
        tot = 0
        for s in range(self.batch):
            n_k = int(self.prompt_lens[s])
            c = int(self.cached_lens[s])
            n = n_k - c
            pairs = n * c + n * (n + 1) // 2 if self.causal else n * n_k
            tot += pairs
        return 4 * self.head_dim * self.num_q_heads * tot


def _scatter_tokens(cache: torch.Tensor, bt_row: np.ndarray, src: torch.Tensor, first: int, B: int):
    """Write src (tokens first..first+len-1 of one sequence) into the paged cache."""
    n = src.shape[0]
    p = 0
    while p < n:
        pos = first + p
        blk = int(bt_row[pos // B])
        off = pos % B
        take = min(B - off, n - p)
        cache[blk, off:off + take] = src[p:p + take]
        p += take


def _slots(bt_row: np.ndarray, first: int, count: int, B: int) -> np.ndarray:
    pos = np.arange(first, first + count, dtype=np.int64)
    return (bt_row[pos // B].astype(np.int64) * B + pos % B).astype(np.int32)


def _poison_uncovered(k_cache, v_cache, block_table, covered_lens, B, poison, rng):
    """Fill every slot outside [0, covered_len) of each sequence (and unused blocks)."""
    nb = k_cache.shape[0]
    covered = np.zeros((nb, B), dtype=bool)
    for s in range(block_table.shape[0]):
        n = int(covered_lens[s])
        for i in range((n + B - 1) // B):
            covered[int(block_table[s, i]), :min(B, n - i * B)] = True
    mask = torch.from_numpy(~covered)
    if not bool(mask.any()):
        return
    fill_shape = (int(mask.sum()),) + tuple(k_cache.shape[2:])
    k_cache[mask] = _fill_bf16(fill_shape, poison, rng)
    v_cache[mask] = _fill_bf16(fill_shape, poison, rng)


def make_decode_case(context_lens, num_q_heads, num_kv_heads, head_dim, block_size,
                     num_blocks=None, seed=0, poison=True, shared_prefix_blocks=0,
                     keep_contiguous=True, name="decode", softmax_scale=None) -> DecodeCase:
    """Build one decode step.

    Each sequence s holds context_lens[s] tokens after this step's store:
    tokens 0..ctx-2 are history already in the cache, token ctx-1 is the new
    row (k_new / v_new) whose slot is ``slot_mapping[s]``.  With
    ``shared_prefix_blocks = P`` every sequence's first P logical blocks map
    to the same P physical blocks (a prefix-cache hit); those tokens are drawn
    once and contexts must extend past them.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    ctx = np.asarray(context_lens, dtype=np.int32)
    batch = ctx.shape[0]
    B = block_size
    Hkv, D = num_kv_heads, head_dim
    assert num_q_heads % num_kv_heads == 0
    assert (ctx >= 1).all()
    nblk = (ctx.astype(np.int64) + B - 1) // B
    P = shared_prefix_blocks
    if P:
        assert (ctx > P * B).all(), "contexts must extend past the shared prefix"
    needed = int(nblk.sum()) - (batch - 1) * P if P else int(nblk.sum())
    if num_blocks is None:
        num_blocks = _with_slack(needed)
    assert num_blocks >= needed
    perm = rng.permutation(num_blocks).astype(np.int32)
    max_blocks = int(nblk.max()) if batch else 1
    block_table = np.full((batch, max_blocks), -1, dtype=np.int32)
    nxt = 0
    shared_ids = perm[:P]
    nxt = P
    for s in range(batch):
        block_table[s, :P] = shared_ids
        k = int(nblk[s]) - P
        block_table[s, P:P + k] = perm[nxt:nxt + k]
        nxt += k

    k_cache = torch.empty((num_blocks, B, Hkv, D), dtype=torch.bfloat16)
    v_cache = torch.empty_like(k_cache)
    k_new = torch.empty((batch, Hkv, D), dtype=torch.bfloat16)
    v_new = torch.empty_like(k_new)
    k_seq, v_seq = ([], []) if keep_contiguous else (None, None)
    shared_k = shared_v = None
    if P:
        shared_k = _normal_bf16(rng, (P * B, Hkv, D))
        shared_v = _normal_bf16(rng, (P * B, Hkv, D))
        _scatter_tokens(k_cache, block_table[0], shared_k, 0, B)
        _scatter_tokens(v_cache, block_table[0], shared_v, 0, B)
    for s in range(batch):
        n = int(ctx[s])
        own = n - P * B
        ks = _normal_bf16(rng, (own, Hkv, D))
        vs = _normal_bf16(rng, (own, Hkv, D))
        # history (all but the newest token) goes into the cache now;
        # the newest token is this step's store.
        _scatter_tokens(k_cache, block_table[s], ks[:own - 1], P * B, B)
        _scatter_tokens(v_cache, block_table[s], vs[:own - 1], P * B, B)
        k_new[s] = ks[own - 1]
        v_new[s] = vs[own - 1]
        if keep_contiguous:
            if P:
                k_seq.append(torch.cat([shared_k, ks]))
                v_seq.append(torch.cat([shared_v, vs]))
            else:
                k_seq.append(ks)
                v_seq.append(vs)
    _poison_uncovered(k_cache, v_cache, block_table, ctx - 1, B, poison, rng)
    slot_mapping = np.array([_slots(block_table[s], int(ctx[s]) - 1, 1, B)[0] for s in range(batch)],
                            dtype=np.int32)
    q = _normal_bf16(rng, (batch, num_q_heads, D))
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    return DecodeCase(name=name, seed=seed, num_q_heads=num_q_heads, num_kv_heads=Hkv, head_dim=D,
                      block_size=B, num_blocks=num_blocks, context_lens=ctx, block_table=block_table,
                      k_cache=k_cache, v_cache=v_cache, k_new=k_new, v_new=v_new,
                      slot_mapping=slot_mapping, q=q, softmax_scale=float(softmax_scale),
                      k_seq=k_seq, v_seq=v_seq, shared_prefix_blocks=P)


def _ramp_keys(ks: torch.Tensor, key_growth: float) -> torch.Tensor:
    """Scale the K row at position p by 1 + key_growth * p / 128 (rounded back to bf16), so that the
    attention scores of later keys spread ever wider: the running maximum of a query's scores keeps
    rising along the sequence.  key_growth = 0 returns the rows untouched."""
    if not key_growth:
        return ks
    ramp = 1.0 + key_growth * torch.arange(ks.shape[0], dtype=torch.float32) / 128.0
    return (ks.float() * ramp[:, None, None]).to(torch.bfloat16)


def make_prefill_case(prompt_lens, cached_lens, num_q_heads, num_kv_heads, head_dim, block_size,
                      num_blocks=None, seed=0, poison=True, keep_contiguous=True, causal=True,
                      name="prefill", softmax_scale=None, key_growth=0.0) -> PrefillCase:
    """Build one varlen prefill step.

    Sequence s has prompt_lens[s] tokens; its first cached_lens[s] tokens (a
    whole number of blocks) already sit in the cache from a prefix-cache hit,
    the remaining n_new = prompt_len - cached_len tokens are stored this step
    and are the queries.  ``key_growth`` > 0 scales the K row at position p
    by 1 + key_growth * p / 128 (see ``_ramp_keys``); it draws no extra random
    numbers, so the other values are those of the same seed without it.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    L = np.asarray(prompt_lens, dtype=np.int32)
    c = np.asarray(cached_lens, dtype=np.int32)
    batch = L.shape[0]
    B = block_size
    Hkv, D = num_kv_heads, head_dim
    assert num_q_heads % num_kv_heads == 0
    assert ((c % B) == 0).all() and (c <= L).all() and (c >= 0).all()
    n_new = L - c
    nblk = (L.astype(np.int64) + B - 1) // B
    needed = int(nblk.sum())
    if num_blocks is None:
        num_blocks = max(1, _with_slack(needed))
    perm = rng.permutation(num_blocks).astype(np.int32)
    max_blocks = max(1, int(nblk.max()) if batch else 1)
    block_table = np.full((batch, max_blocks), -1, dtype=np.int32)
    nxt = 0
    for s in range(batch):
        k = int(nblk[s])
        block_table[s, :k] = perm[nxt:nxt + k]
        nxt += k
    k_cache = torch.empty((num_blocks, B, Hkv, D), dtype=torch.bfloat16)
    v_cache = torch.empty_like(k_cache)
    total_q = int(n_new.sum())
    k_new = torch.empty((total_q, Hkv, D), dtype=torch.bfloat16)
    v_new = torch.empty_like(k_new)
    cu_q = np.zeros(batch + 1, dtype=np.int32)
    cu_k = np.zeros(batch + 1, dtype=np.int32)
    cu_q[1:] = np.cumsum(n_new)
    cu_k[1:] = np.cumsum(L)
    slot_mapping = np.empty(total_q, dtype=np.int32)
    k_seq, v_seq = ([], []) if keep_contiguous else (None, None)
    for s in range(batch):
        n = int(L[s])
        ks = _ramp_keys(_normal_bf16(rng, (n, Hkv, D)), key_growth)
        vs = _normal_bf16(rng, (n, Hkv, D))
        cs = int(c[s])
        _scatter_tokens(k_cache, block_table[s], ks[:cs], 0, B)
        _scatter_tokens(v_cache, block_table[s], vs[:cs], 0, B)
        a, b = int(cu_q[s]), int(cu_q[s + 1])
        k_new[a:b] = ks[cs:]
        v_new[a:b] = vs[cs:]
        slot_mapping[a:b] = _slots(block_table[s], cs, n - cs, B)
        if keep_contiguous:
            k_seq.append(ks)
            v_seq.append(vs)
    _poison_uncovered(k_cache, v_cache, block_table, c, B, poison, rng)
    q = _normal_bf16(rng, (total_q, num_q_heads, D))
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    return PrefillCase(name=name, seed=seed, num_q_heads=num_q_heads, num_kv_heads=Hkv, head_dim=D,
                       block_size=B, num_blocks=num_blocks, prompt_lens=L, cached_lens=c,
                       cu_seqlens_q=cu_q, cu_seqlens_k=cu_k, block_table=block_table,
                       k_cache=k_cache, v_cache=v_cache, k_new=k_new, v_new=v_new,
                       slot_mapping=slot_mapping, q=q, softmax_scale=float(softmax_scale),
                       causal=causal, k_seq=k_seq, v_seq=v_seq)


# ---------------------------------------------------------------------------
# The five workloads: shapes from the pages' Qwen-class serving setups.
# ---------------------------------------------------------------------------

def tiny_decode(poison=True, keep_contiguous=True) -> DecodeCase:
    """Batch 4, contexts {1,17,100,255}, 4 q / 2 kv heads, head_dim 64, block 16, 64 blocks."""
    return make_decode_case([1, 17, 100, 255], 4, 2, 64, 16, num_blocks=64, seed=1001,
                            poison=poison, keep_contiguous=keep_contiguous, name="tiny_decode")


def qwen3_06b_decode(poison=True, keep_contiguous=True) -> DecodeCase:
    """Qwen3-0.6B-like: batch 64, contexts U{100..1024}, 16 q / 8 kv heads, D 128, block 256."""
    rng = np.random.Generator(np.random.PCG64(1002))
    ctx = rng.integers(100, 1025, size=64).astype(np.int32)
    return make_decode_case(ctx, 16, 8, 128, 256, seed=2002, poison=poison,
                            keep_contiguous=keep_contiguous, name="qwen3_0.6b_decode")


def long_context_decode(poison=True, keep_contiguous=False) -> DecodeCase:
    """Batch 8, context 32768 each, 32 q / 8 kv heads, D 128, block 256."""
    return make_decode_case([32768] * 8, 32, 8, 128, 256, seed=1003, poison=poison,
                            keep_contiguous=keep_contiguous, name="long_context_decode")


def prefix_sharing_decode(poison=True, keep_contiguous=False) -> DecodeCase:
    """256 sequences sharing 16 physical blocks (4096 tokens) plus private suffixes.

    Each sequence has s ~ U{0..512} private tokens already cached plus the new
    token stored this step, so its context is 4096 + s + 1.
    """
    rng = np.random.Generator(np.random.PCG64(1004))
    priv = rng.integers(0, 513, size=256).astype(np.int32)
    ctx = 4096 + priv + 1
    return make_decode_case(ctx, 16, 8, 128, 256, seed=2004, poison=poison, shared_prefix_blocks=16,
                            keep_contiguous=keep_contiguous, name="prefix_sharing_decode")


def varlen_prefill(poison=True, keep_contiguous=False) -> PrefillCase:
    """12 prompts of U{128..2048} tokens, 32 q / 8 kv heads, D 128, block 256.

    Prompts 0, 2, ..., 10 have a cached prefix of 256*u tokens,
    u ~ U{1..floor((L-1)/256)} (0 when L <= 256), so at least one new token
    is left to compute.
    """
    rng = np.random.Generator(np.random.PCG64(1005))
    L = rng.integers(128, 2049, size=12).astype(np.int32)
    c = np.zeros(12, dtype=np.int32)
    for s in range(0, 12, 2):
        umax = (int(L[s]) - 1) // 256
        c[s] = 256 * int(rng.integers(1, umax + 1)) if umax >= 1 else 0
    return make_prefill_case(L, c, 32, 8, 128, 256, seed=2005, poison=poison,
                             keep_contiguous=keep_contiguous, name="varlen_prefill")


WORKLOADS = {
    "tiny_decode": tiny_decode,
    "qwen3_0.6b_decode": qwen3_06b_decode,
    "long_context_decode": long_context_decode,
    "prefix_sharing_decode": prefix_sharing_decode,
    "varlen_prefill": varlen_prefill,
}
