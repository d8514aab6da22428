"""Seeded synthetic inputs for paged-KV attention.

This module draws numbers and lays them out. It has none of the attention
arithmetic: no dot products, no softmax, no gather for compute. Both the CPU
oracle (``oracle/``) and the CUDA path get their inputs from here, and neither
imports the other.

Layout conventions, from the pages:
  * The KV cache is one physical pool of fixed-size blocks of 16 tokens
    ("vLLM and PagedAttention", ai.zenoagi.com, §2 "The PagedAttention
    Solution"; "vLLM — PagedAttention and Continuous Batching",
    s-samarth.github.io, §2.2).
  * The pool is ``[num_blocks, block_size, num_kv_heads, head_dim]``, following
    the kernel sketch in "vLLM and PagedAttention" §2 "Reworking the Attention
    Computation" (its ``key_cache``/``value_cache`` comment), read with KV heads.
  * Each sequence has a table of physical block ids in logical order. Only its
    last block may be partly filled ("How vLLM Works?", peterindia.net, §03).

The recipe: lengths, layout, values and queries come from four separate numpy
``default_rng`` streams keyed by ``(seed, k)``. Values are drawn U[-1, 1) in
fp32. For bf16 cases they are rounded to bf16 (round to nearest even), and the
oracle uses the rounded values. Free blocks, the unused tail slots of each
last block, and the slots this step's new tokens will go to all hold NaN.
A kernel that reads any of them, or that attends before writing, shows NaN.
Table entries past a sequence's last block are -1.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

BLOCK_SIZE = 16
BF16_NAN_BITS = 0x7FC0

_STREAM_LENGTHS, _STREAM_LAYOUT, _STREAM_VALUES, _STREAM_QUERY = 1, 2, 3, 4


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns the uint16 bit patterns.

    Inputs here are finite, so NaN/Inf handling is not needed.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.asarray(u, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _nan_fill(shape, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return np.full(shape, BF16_NAN_BITS, dtype=np.uint16)
    return np.full(shape, np.nan, dtype=np.float32)


def _uniform(rng: np.random.Generator, shape, dtype: str) -> np.ndarray:
    x = rng.random(shape, dtype=np.float32)
    x *= np.float32(2.0)
    x -= np.float32(1.0)
    return f32_to_bf16_bits(x) if dtype == "bf16" else x


@dataclass
class PagedCase:
    """One step of paged attention: cache before the write, new tokens, queries.

    Shapes (T = total new/query tokens = sum(q_lens)):
      k_cache, v_cache : [num_blocks, block_size, num_kv_heads, head_dim]
      block_tables     : int32 [B, max_blocks_per_seq], -1 past the last block
      context_lens     : int32 [B], length after this step's tokens are appended
      q_lens           : int32 [B], this step's new tokens per sequence
      cu_q_lens        : int32 [B + 1], prefix sums of q_lens
      q                : [T, num_heads, head_dim]
      k_new, v_new     : [T, num_kv_heads, head_dim]
      slot_mapping     : int64 [T], flat slot (block * block_size + offset)
    bf16 arrays hold uint16 bit patterns, f32 arrays hold float32.
    """

    name: str
    seed: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    dtype: str
    scale: float
    num_blocks: int
    context_lens: np.ndarray
    q_lens: np.ndarray
    cu_q_lens: np.ndarray
    block_tables: np.ndarray
    k_cache: np.ndarray
    v_cache: np.ndarray
    q: np.ndarray
    k_new: np.ndarray
    v_new: np.ndarray
    slot_mapping: np.ndarray
    block_size: int = BLOCK_SIZE
    logical_k: Optional[List[np.ndarray]] = field(default=None, repr=False)
    logical_v: Optional[List[np.ndarray]] = field(default=None, repr=False)
    notes: str = ""

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def num_tokens(self) -> int:
        return int(self.cu_q_lens[-1])

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    def kv_bytes_read(self) -> int:
        """K and V bytes one attention pass must read: sum_b c_b * 2 * Hk * D * elem."""
        return int(self.context_lens.astype(np.int64).sum()) * 2 * self.num_kv_heads * self.head_dim * self.elem_bytes


def make_case(
    name: str,
    seed: int,
    *,
    context_lens,
    q_lens,
    num_heads: int,
    num_kv_heads: int,
    head_dim: int,
    dtype: str,
    scale: Optional[float] = None,
    num_blocks: Optional[int] = None,
    pool_factor: float = 1.5,
    shared_prefix_blocks: int = 0,
    copy_shared: bool = False,
    table_slack: int = 0,
    keep_logical: bool = False,
    notes: str = "",
) -> PagedCase:
    """Build one paged step from seeds.

    Sequence b holds logical tokens ``0 .. context_lens[b]-1``. The last
    ``q_lens[b]`` of them are this step's new tokens. The first
    ``shared_prefix_blocks`` logical blocks of every sequence hold the same
    values. They share one set of physical ids unless ``copy_shared`` is set,
    in which case each sequence gets its own copy.
    """
    assert dtype in ("f32", "bf16")
    bs = BLOCK_SIZE
    ctx = np.asarray(context_lens, dtype=np.int64)
    ql = np.asarray(q_lens, dtype=np.int64)
    B = ctx.shape[0]
    assert ql.shape == (B,) and np.all(ql >= 0) and np.all(ql <= ctx)
    nblk = (ctx + bs - 1) // bs
    S = int(shared_prefix_blocks)
    if S:
        assert np.all(nblk >= S) and np.all(ctx - ql >= S * bs), "new tokens must lie past the shared prefix"
    Hk, D = num_kv_heads, head_dim

    private = nblk - S
    needed = int(private.sum()) + (S * B if copy_shared else S)
    if num_blocks is None:
        num_blocks = max(int(math.ceil(pool_factor * needed)), needed)
    assert num_blocks >= needed

    rng_layout = np.random.default_rng([seed, _STREAM_LAYOUT])
    rng_vals = np.random.default_rng([seed, _STREAM_VALUES])
    rng_q = np.random.default_rng([seed, _STREAM_QUERY])

    perm = rng_layout.permutation(num_blocks).astype(np.int32)
    MB = int(nblk.max()) + int(table_slack) if B else 1
    tables = np.full((B, max(MB, 1)), -1, dtype=np.int32)
    cursor = 0
    shared_ids = None
    if S and not copy_shared:
        shared_ids = perm[cursor:cursor + S]
        cursor += S
    for b in range(B):
        if S:
            if copy_shared:
                tables[b, :S] = perm[cursor:cursor + S]
                cursor += S
            else:
                tables[b, :S] = shared_ids
        n = int(private[b])
        tables[b, S:S + n] = perm[cursor:cursor + n]
        cursor += n

    k_cache = _nan_fill((num_blocks, bs, Hk, D), dtype)
    v_cache = _nan_fill((num_blocks, bs, Hk, D), dtype)

    shared_k = shared_v = None
    if S:
        shared_k = _uniform(rng_vals, (S, bs, Hk, D), dtype)
        shared_v = _uniform(rng_vals, (S, bs, Hk, D), dtype)
        if copy_shared:
            for b in range(B):
                k_cache[tables[b, :S]] = shared_k
                v_cache[tables[b, :S]] = shared_v
        else:
            k_cache[shared_ids] = shared_k
            v_cache[shared_ids] = shared_v

    T = int(ql.sum())
    cu = np.zeros(B + 1, dtype=np.int32)
    cu[1:] = np.cumsum(ql)
    k_new = np.empty((T, Hk, D), dtype=k_cache.dtype)
    v_new = np.empty((T, Hk, D), dtype=v_cache.dtype)
    slots = np.empty(T, dtype=np.int64)
    logical_k = [] if keep_logical else None
    logical_v = [] if keep_logical else None
    poison = BF16_NAN_BITS if dtype == "bf16" else np.float32(np.nan)

    for b in range(B):
        n = int(private[b])
        pk = _uniform(rng_vals, (n, bs, Hk, D), dtype)
        pv = _uniform(rng_vals, (n, bs, Hk, D), dtype)
        ids = tables[b, S:S + n]
        # logical block S+i of sequence b lives in physical block ids[i]
        k_cache[ids] = pk
        v_cache[ids] = pv
        c = int(ctx[b])
        if keep_logical:
            parts_k = ([shared_k.reshape(S * bs, Hk, D)] if S else []) + [pk.reshape(n * bs, Hk, D)]
            parts_v = ([shared_v.reshape(S * bs, Hk, D)] if S else []) + [pv.reshape(n * bs, Hk, D)]
            logical_k.append(np.concatenate(parts_k, axis=0)[:c].copy())
            logical_v.append(np.concatenate(parts_v, axis=0)[:c].copy())
        # unused tail slots of the last block are poison
        if n and c % bs:
            last = ids[-1]
            k_cache[last, c % bs:] = poison
            v_cache[last, c % bs:] = poison
        # this step's tokens: move their values out of the pool, poison the slots
        t0 = int(cu[b])
        for j in range(int(ql[b])):
            p = c - int(ql[b]) + j
            li = p // bs - S
            off = p % bs
            k_new[t0 + j] = pk[li, off]
            v_new[t0 + j] = pv[li, off]
            slots[t0 + j] = int(ids[li]) * bs + off
        if ql[b]:
            flat_k = k_cache.reshape(-1, Hk, D)
            flat_v = v_cache.reshape(-1, Hk, D)
            flat_k[slots[t0:t0 + int(ql[b])]] = poison
            flat_v[slots[t0:t0 + int(ql[b])]] = poison

    q = _uniform(rng_q, (T, num_heads, D), dtype)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    return PagedCase(
        name=name, seed=seed, num_heads=num_heads, num_kv_heads=Hk, head_dim=D, dtype=dtype,
        scale=float(scale), num_blocks=int(num_blocks), context_lens=ctx.astype(np.int32),
        q_lens=ql.astype(np.int32), cu_q_lens=cu, block_tables=tables, k_cache=k_cache,
        v_cache=v_cache, q=q, k_new=k_new, v_new=v_new, slot_mapping=slots,
        logical_k=logical_k, logical_v=logical_v, notes=notes,
    )


# ---------------------------------------------------------------------------
# The five serving-shaped workloads.

def tiny(seed: int = 0, keep_logical: bool = True) -> PagedCase:
    """4 sequences, 4 query heads / 1 KV head, head_dim 64, fp32, lengths {1,15,16,37}.

    Pool of 16 blocks. Tables are a random pick of distinct pool blocks. One
    spare table column is -1.
    """
    return make_case("tiny", seed, context_lens=[1, 15, 16, 37], q_lens=[1, 1, 1, 1], num_heads=4,
                     num_kv_heads=1, head_dim=64, dtype="f32", scale=1.0 / 8.0, num_blocks=16,
                     table_slack=1, keep_logical=keep_logical)


def decode_batch(seed: int = 1, keep_logical: bool = False) -> PagedCase:
    """64 sequences, 32/8 heads, head_dim 128, bf16, lengths U{128..2048}, pool 1.5x needed."""
    rng = np.random.default_rng([seed, _STREAM_LENGTHS])
    ctx = rng.integers(128, 2048, size=64, endpoint=True)
    return make_case("decode_batch", seed, context_lens=ctx, q_lens=np.ones(64, np.int64), num_heads=32,
                     num_kv_heads=8, head_dim=128, dtype="bf16", keep_logical=keep_logical)


def long_context(seed: int = 2, keep_logical: bool = False) -> PagedCase:
    """8 sequences of 32768 tokens (2048 blocks each), 32/8 heads, head_dim 128, bf16, pool 24576 blocks."""
    return make_case("long_context", seed, context_lens=[32768] * 8, q_lens=[1] * 8, num_heads=32,
                     num_kv_heads=8, head_dim=128, dtype="bf16", num_blocks=24576,
                     keep_logical=keep_logical)


PREFIX_SHARED_BLOCKS = 94  # 1504 tokens = 94 full blocks


def prefix_sharing(seed: int = 3, copy_shared: bool = False, keep_logical: bool = False) -> PagedCase:
    """256 sequences: a 1504-token prefix (94 full blocks) plus private tails of U{8..512} tokens.

    With ``copy_shared`` False every table points at the same 94 physical
    blocks. With it True each sequence has its own copy of them. Logical
    contents are identical either way.
    """
    rng = np.random.default_rng([seed, _STREAM_LENGTHS])
    tails = rng.integers(8, 512, size=256, endpoint=True)
    ctx = PREFIX_SHARED_BLOCKS * BLOCK_SIZE + tails
    return make_case("prefix_sharing" + ("_copied" if copy_shared else ""), seed, context_lens=ctx,
                     q_lens=np.ones(256, np.int64), num_heads=32, num_kv_heads=8, head_dim=128,
                     dtype="bf16", shared_prefix_blocks=PREFIX_SHARED_BLOCKS, copy_shared=copy_shared,
                     keep_logical=keep_logical)


def mixed_step(seed: int = 4, keep_logical: bool = False) -> PagedCase:
    """One causal prefill chunk (2048 query tokens at offset 6144) plus 192 decode sequences.

    Decode lengths are U{256..4096}. 32/8 heads, head_dim 128, bf16, 2240 new
    tokens in all. Sequence 0 is the prefill, sequences 1..192 are decodes.
    """
    rng = np.random.default_rng([seed, _STREAM_LENGTHS])
    dec = rng.integers(256, 4096, size=192, endpoint=True)
    ctx = np.concatenate([[8192], dec])
    ql = np.concatenate([[2048], np.ones(192, np.int64)])
    return make_case("mixed_step", seed, context_lens=ctx, q_lens=ql, num_heads=32, num_kv_heads=8,
                     head_dim=128, dtype="bf16", keep_logical=keep_logical)


def prefill_chunk(seed: int = 4, keep_logical: bool = False) -> PagedCase:
    """The mixed step's prefill alone: one sequence, 2048 query tokens at offset 6144 (c = 8192)."""
    return make_case("prefill_chunk", seed, context_lens=[8192], q_lens=[2048], num_heads=32, num_kv_heads=8,
                     head_dim=128, dtype="bf16", keep_logical=keep_logical)


def spec_verify(seed: int = 5, keep_logical: bool = False) -> PagedCase:
    """64 sequences each verifying a chunk of 4 tokens (3 drafted + 1), the decode batch's shape otherwise.

    Lengths U{128..2048} after the append, 32/8 heads, head_dim 128, bf16,
    256 new tokens in all.
    """
    rng = np.random.default_rng([seed, _STREAM_LENGTHS])
    ctx = rng.integers(128, 2048, size=64, endpoint=True)
    return make_case("spec_verify", seed, context_lens=ctx, q_lens=np.full(64, 4, np.int64), num_heads=32,
                     num_kv_heads=8, head_dim=128, dtype="bf16", keep_logical=keep_logical)


CONFIGS = {
    "tiny": tiny,
    "decode_batch": decode_batch,
    "long_context": long_context,
    "prefix_sharing": prefix_sharing,
    "mixed_step": mixed_step,
    "prefill_chunk": prefill_chunk,
    "spec_verify": spec_verify,
}
