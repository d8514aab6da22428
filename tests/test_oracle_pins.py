"""Pins for the fp64 oracle. CPU only, so none of these is marked gpu.

Each pin checks the oracle against something other than itself:
  * the worked examples the pages print (tests/golden/page_examples.txt),
  * torch's scaled_dot_product_attention in fp64 (a library routine) on the
    contiguous K/V the generator drew before paging them,
  * closed forms: one token gives its V row, identical keys give the mean of V,
    a dominant key gives its V row,
  * invariants: permuting physical blocks, or copying shared blocks, leaves
    the output bit-identical.
test_planted_mistakes_are_caught plants each mistake of the oracle's mutation
list and checks that at least one pin fails.
"""
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from paged_kv_cache_366_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_examples.txt")
TOL = 1e-12


def widen(a):
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return W.bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


def read_golden():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                key, *vals = line.split()
                rows.append((key, [int(v) for v in vals]))
    return rows


def written(case):
    """Cache after this step's write, by the oracle's write."""
    return oracle.reshape_and_cache(case.k_new, case.v_new, case.k_cache, case.v_cache, case.slot_mapping)


def sdpa_decode(case):
    """Library attention on the generator's contiguous K/V, one query per sequence."""
    G = case.num_heads // case.num_kv_heads
    out = np.zeros((case.num_seqs, case.num_heads, case.head_dim))
    for b in range(case.num_seqs):
        c = int(case.context_lens[b])
        if c == 0:
            continue
        q = torch.from_numpy(widen(case.q[case.cu_q_lens[b + 1] - 1]))[None, :, None, :]
        k = torch.from_numpy(widen(case.logical_k[b])).permute(1, 0, 2)[None]
        v = torch.from_numpy(widen(case.logical_v[b])).permute(1, 0, 2)[None]
        o = F.scaled_dot_product_attention(q, k, v, scale=case.scale, enable_gqa=G > 1)
        out[b] = o[0, :, 0, :].numpy()
    return out


def sdpa_prefill(case):
    """Library attention with an explicit causal mask at each chunk's offset."""
    out = np.zeros((case.num_tokens, case.num_heads, case.head_dim))
    G = case.num_heads // case.num_kv_heads
    for b in range(case.num_seqs):
        q0, q1 = int(case.cu_q_lens[b]), int(case.cu_q_lens[b + 1])
        c = int(case.context_lens[b])
        if q1 == q0:
            continue
        off = c - (q1 - q0)
        q = torch.from_numpy(widen(case.q[q0:q1])).permute(1, 0, 2)[None]
        k = torch.from_numpy(widen(case.logical_k[b])).permute(1, 0, 2)[None]
        v = torch.from_numpy(widen(case.logical_v[b])).permute(1, 0, 2)[None]
        pos = off + torch.arange(q1 - q0)[:, None]
        mask = torch.arange(c)[None, :] <= pos
        o = F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=case.scale, enable_gqa=G > 1)
        out[q0:q1] = o[0].permute(1, 0, 2).numpy()
    return out


def small_decode_case(seed, H=8, Hk=2, D=64, dtype="f32", ctx=(1, 15, 16, 17, 37, 100), **kw):
    return W.make_case("pin", seed, context_lens=list(ctx), q_lens=[1] * len(ctx), num_heads=H,
                       num_kv_heads=Hk, head_dim=D, dtype=dtype, scale=kw.pop("scale", 0.37),
                       keep_logical=True, table_slack=1, **kw)


def small_prefill_case(seed, H=8, Hk=2, D=64, dtype="f32", ctx=(40, 33, 70), ql=(40, 9, 17), **kw):
    return W.make_case("pin_prefill", seed, context_lens=list(ctx), q_lens=list(ql), num_heads=H,
                       num_kv_heads=Hk, head_dim=D, dtype=dtype, scale=kw.pop("scale", 0.29),
                       keep_logical=True, **kw)


# ---------------------------------------------------------------------------
# Pins, as plain functions so the planted-mistake test can run them all.

def pin_page_block_arithmetic():
    bs = 16
    for key, vals in read_golden():
        if key == "block_size":
            bs = vals[0]
        elif key == "blocks_for":
            assert oracle.blocks_for(vals[0], bs) == vals[1], (key, vals)
        elif key == "position_block_offset":
            pos, blk, off = vals
            table = np.arange(1000, 1000 + blk + 2, dtype=np.int32)
            assert oracle.slot_of(table, pos, bs) == int(table[blk]) * bs + off


def pin_page_tables_gather():
    """Mark every pool row with (block id, row); gathering through a page table reads them back in order."""
    bs = 16
    for key, vals in read_golden():
        if key != "table":
            continue
        table = np.array([vals], dtype=np.int32)
        nb = max(vals) + 1
        kc = np.zeros((nb, bs, 1, 2), np.float32)
        kc[:, :, 0, 0] = np.arange(nb)[:, None]
        kc[:, :, 0, 1] = np.arange(bs)[None, :]
        vc = -kc
        n = len(vals) * bs - 5  # last block partly filled
        K, V = oracle.gather(kc, vc, table, 0, n, 0, bs)
        for p in range(n):
            assert K[p, 0] == vals[p // bs] and K[p, 1] == p % bs, (vals, p, K[p])
            assert V[p, 0] == -vals[p // bs]


def pin_decode_matches_library(dtype="f32", H=8, Hk=2, D=64, seed=11):
    case = small_decode_case(seed, H=H, Hk=Hk, D=D, dtype=dtype)
    kc, vc = written(case)
    got = oracle.decode(case.q, kc, vc, case.block_tables, case.context_lens, case.scale)
    ref = sdpa_decode(case)
    err = np.abs(got - ref).max()
    assert err <= TOL, err


def pin_tiny_config_matches_library():
    case = W.tiny()
    kc, vc = written(case)
    got = oracle.decode(case.q, kc, vc, case.block_tables, case.context_lens, case.scale)
    err = np.abs(got - sdpa_decode(case)).max()
    assert err <= TOL, err


def pin_block_permutation_invariant():
    case = small_decode_case(21, dtype="bf16", D=128)
    kc, vc = written(case)
    base = oracle.decode(case.q, kc, vc, case.block_tables, case.context_lens, case.scale)
    perm = np.random.default_rng(5).permutation(case.num_blocks)
    kc2 = np.empty_like(kc)
    vc2 = np.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    bt2 = np.where(case.block_tables >= 0, perm[np.maximum(case.block_tables, 0)], -1).astype(np.int32)
    moved = oracle.decode(case.q, kc2, vc2, bt2, case.context_lens, case.scale)
    assert np.array_equal(base, moved)


def pin_single_token_gives_its_value_row():
    case = small_decode_case(31, ctx=(1, 1, 1))
    kc, vc = written(case)
    out = oracle.decode(case.q, kc, vc, case.block_tables, case.context_lens, case.scale)
    G = case.num_heads // case.num_kv_heads
    for b in range(case.num_seqs):
        for h in range(case.num_heads):
            assert np.array_equal(out[b, h], widen(case.v_new[b, h // G]))


def pin_identical_keys_give_mean_value():
    case = small_decode_case(41, ctx=(5, 16, 37))
    kc, vc = written(case)
    # every key of every sequence and head is the same vector
    kc = kc.copy()
    kc[...] = np.float32(0.25)
    out = oracle.decode(case.q, kc, vc, case.block_tables, case.context_lens, case.scale)
    G = case.num_heads // case.num_kv_heads
    for b in range(case.num_seqs):
        for h in range(case.num_heads):
            mean_v = widen(case.logical_v[b][:, h // G]).mean(axis=0)
            assert np.abs(out[b, h] - mean_v).max() <= TOL


def pin_dominant_key_gives_its_value_row():
    case = small_decode_case(51, ctx=(37,), H=2, Hk=2, scale=1.0e3)
    kc, vc = written(case)
    kc = kc.copy()
    q = np.zeros_like(case.q)
    q[:, :, 0] = 1.0
    kc[...] = 0.0
    j = 29
    slot = oracle.slot_of(case.block_tables[0], j)
    kc.reshape(-1, case.num_kv_heads, case.head_dim)[slot, :, 0] = 1.0
    out = oracle.decode(q, kc, vc, case.block_tables, case.context_lens, case.scale)
    for h in range(case.num_heads):
        assert np.abs(out[0, h] - widen(case.logical_v[0][j, h])).max() <= TOL


def pin_shared_prefix_equals_copies():
    kw = dict(context_lens=[3 * 16 + 5, 3 * 16 + 20, 3 * 16 + 1, 3 * 16 + 16], q_lens=[1] * 4, num_heads=8,
              num_kv_heads=2, head_dim=64, dtype="bf16", shared_prefix_blocks=3)
    a = W.make_case("shared", 61, copy_shared=False, **kw)
    b = W.make_case("copied", 61, copy_shared=True, **kw)
    assert len(np.unique(a.block_tables[:, :3])) == 3 and len(np.unique(b.block_tables[:, :3])) == 12
    ka, va = written(a)
    kb, vb = written(b)
    oa = oracle.decode(a.q, ka, va, a.block_tables, a.context_lens, a.scale)
    ob = oracle.decode(b.q, kb, vb, b.block_tables, b.context_lens, b.scale)
    assert np.array_equal(oa, ob)


def pin_prefill_offset_zero_is_causal_attention():
    case = small_prefill_case(71, ctx=(40, 23), ql=(40, 23))
    kc, vc = written(case)
    got = oracle.prefill(case.q, kc, vc, case.block_tables, case.cu_q_lens, case.context_lens, case.scale)
    # textbook causal attention, no offset: is_causal on square blocks
    for b in range(case.num_seqs):
        q0, q1 = int(case.cu_q_lens[b]), int(case.cu_q_lens[b + 1])
        q = torch.from_numpy(widen(case.q[q0:q1])).permute(1, 0, 2)[None]
        k = torch.from_numpy(widen(case.logical_k[b])).permute(1, 0, 2)[None]
        v = torch.from_numpy(widen(case.logical_v[b])).permute(1, 0, 2)[None]
        o = F.scaled_dot_product_attention(q, k, v, is_causal=True, scale=case.scale, enable_gqa=True)
        assert np.abs(got[q0:q1] - o[0].permute(1, 0, 2).numpy()).max() <= TOL


def pin_prefill_at_offset_matches_library(dtype="f32", D=64):
    case = small_prefill_case(81, dtype=dtype, D=D)
    kc, vc = written(case)
    got = oracle.prefill(case.q, kc, vc, case.block_tables, case.cu_q_lens, case.context_lens, case.scale)
    err = np.abs(got - sdpa_prefill(case)).max()
    assert err <= TOL, err


def pin_prefill_single_query_equals_decode():
    case = small_decode_case(91)
    kc, vc = written(case)
    dec = oracle.decode(case.q, kc, vc, case.block_tables, case.context_lens, case.scale)
    pre = oracle.prefill(case.q, kc, vc, case.block_tables, case.cu_q_lens, case.context_lens, case.scale)
    assert np.array_equal(dec, pre)


def pin_write_then_gather_reads_new_tokens():
    case = small_prefill_case(101, dtype="bf16")
    kc, vc = written(case)
    for b in range(case.num_seqs):
        for hk in range(case.num_kv_heads):
            K, V = oracle.gather(kc, vc, case.block_tables, b, int(case.context_lens[b]), hk)
            assert np.array_equal(K, widen(case.logical_k[b][:, hk]))
            assert np.array_equal(V, widen(case.logical_v[b][:, hk]))


def pin_write_leaves_other_bytes():
    case = small_prefill_case(111, dtype="bf16")
    kc, vc = written(case)
    touched = np.zeros(case.num_blocks * 16, bool)
    touched[case.slot_mapping] = True
    before = case.k_cache.reshape(case.num_blocks * 16, -1).view(np.uint8)
    after = kc.reshape(case.num_blocks * 16, -1).view(np.uint8)
    assert np.array_equal(before[~touched], after[~touched])
    assert np.array_equal(after[case.slot_mapping], case.k_new.reshape(len(case.slot_mapping), -1).view(np.uint8))


def pin_write_page_example_slot():
    """The 100th token of a sequence goes to row 3 of its 7th block's physical id."""
    table = np.array([[42, 17, 5, 99, 31, 7, 60, 3]], np.int32)
    nb = 100
    kc = np.zeros((nb, 16, 1, 4), np.float32)
    vc = np.zeros_like(kc)
    slot = oracle.slot_of(table[0], 99)
    k = np.full((1, 1, 4), 7.0, np.float32)
    kc2, _ = oracle.reshape_and_cache(k, -k, kc, vc, np.array([slot], np.int64))
    assert np.all(kc2[60, 3] == 7.0) and np.count_nonzero(kc2) == 4


PINS = [
    pin_page_block_arithmetic,
    pin_page_tables_gather,
    pin_decode_matches_library,
    pin_tiny_config_matches_library,
    pin_block_permutation_invariant,
    pin_single_token_gives_its_value_row,
    pin_identical_keys_give_mean_value,
    pin_dominant_key_gives_its_value_row,
    pin_shared_prefix_equals_copies,
    pin_prefill_offset_zero_is_causal_attention,
    pin_prefill_at_offset_matches_library,
    pin_prefill_single_query_equals_decode,
    pin_write_then_gather_reads_new_tokens,
    pin_write_leaves_other_bytes,
    pin_write_page_example_slot,
]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    assert oracle.get_mutation() == 0
    pin()


@pytest.mark.parametrize("dtype,H,Hk,D", [("f32", 4, 4, 64), ("f32", 8, 1, 128), ("bf16", 32, 8, 128),
                                          ("bf16", 6, 3, 64)])
def test_decode_matches_library_shapes(dtype, H, Hk, D):
    pin_decode_matches_library(dtype=dtype, H=H, Hk=Hk, D=D, seed=hash((dtype, H, Hk, D)) % 1000)


def test_prefill_matches_library_bf16():
    pin_prefill_at_offset_matches_library(dtype="bf16", D=128)


def test_write_negative_slot_is_skipped():
    case = small_decode_case(121)
    slots = case.slot_mapping.copy()
    slots[1] = -1
    kc, vc = oracle.reshape_and_cache(case.k_new, case.v_new, case.k_cache, case.v_cache, slots)
    flat = kc.reshape(case.num_blocks * 16, -1)
    assert np.all(np.isnan(flat[case.slot_mapping[1]]))
    assert np.array_equal(flat[slots[0]], case.k_new[0].reshape(-1))


def test_write_rejects_slot_outside_pool():
    case = small_decode_case(131)
    slots = case.slot_mapping.copy()
    slots[0] = case.num_blocks * 16
    with pytest.raises(oracle.OracleError):
        oracle.reshape_and_cache(case.k_new, case.v_new, case.k_cache, case.v_cache, slots)


def test_zero_context_gives_zeros():
    case = small_decode_case(141, ctx=(1, 5))
    kc, vc = written(case)
    lens = case.context_lens.copy()
    lens[0] = 0
    out = oracle.decode(case.q, kc, vc, case.block_tables, lens, case.scale)
    assert np.all(out[0] == 0.0) and np.all(np.isfinite(out[1]))


def test_unused_entries_are_never_read():
    """Every value the oracle reads is finite, although free blocks, tails and spare table entries are poison."""
    case = small_decode_case(151, dtype="bf16")
    assert np.any(case.block_tables == -1)
    kc, vc = written(case)
    out = oracle.decode(case.q, kc, vc, case.block_tables, case.context_lens, case.scale)
    assert np.all(np.isfinite(out))


def test_attending_before_the_write_shows_poison():
    case = small_decode_case(161)
    out = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale)
    assert np.all(np.isnan(out))


def test_prefill_row_subset_matches_full():
    case = small_prefill_case(171)
    kc, vc = written(case)
    full = oracle.prefill(case.q, kc, vc, case.block_tables, case.cu_q_lens, case.context_lens, case.scale)
    rows = np.array([0, 5, 39, 40, 48, 49, 65], np.int32)
    sub = oracle.prefill(case.q, kc, vc, case.block_tables, case.cu_q_lens, case.context_lens, case.scale,
                         rows=rows)
    assert np.array_equal(sub, full[rows])


MUTATIONS = list(range(1, 11))


@pytest.mark.parametrize("mutation", MUTATIONS)
def test_planted_mistakes_are_caught(mutation):
    failures = []
    oracle.set_mutation(mutation)
    try:
        for pin in PINS:
            try:
                pin()
            except (AssertionError, oracle.OracleError) as e:
                failures.append(pin.__name__)
    finally:
        oracle.set_mutation(0)
    assert failures, "mutation %d passed every pin" % mutation


# ---------------------------------------------------------------------------
# Block copies (copy-on-write fork, swap out/in), pinned by the attention they preserve.

def _fork_case(seed=181):
    # two sequences sharing all three blocks of a 37-token prefix; each appends one token
    return W.make_case("fork", seed, context_lens=[37, 37], q_lens=[0, 0], num_heads=8, num_kv_heads=2,
                       head_dim=64, dtype="f32", shared_prefix_blocks=2, keep_logical=True, table_slack=1)


def test_copy_on_write_fork_keeps_sequences_apart():
    """After copying the shared last block for sequence 1 and writing each sequence's
    next token into its own last block, each sequence attends to its own token."""
    case = _fork_case()
    bt = case.block_tables.copy()
    bt[1, :3] = bt[0, :3]  # sequence 1 shares all of sequence 0's blocks, the partial last one too
    kc, vc = case.k_cache.copy(), case.v_cache.copy()
    free = np.setdiff1d(np.arange(case.num_blocks), bt[bt >= 0])
    new_blk = int(free[0])
    kc, vc = oracle.copy_blocks(kc, vc, [[bt[0, 2], new_blk]])
    bt[1, 2] = new_blk
    rng = np.random.default_rng(3)
    k_tok = rng.uniform(-1, 1, (2, 2, 64)).astype(np.float32)
    v_tok = rng.uniform(-1, 1, (2, 2, 64)).astype(np.float32)
    slots = np.array([oracle.slot_of(bt[0], 37), oracle.slot_of(bt[1], 37)], np.int64)
    kc, vc = oracle.reshape_and_cache(k_tok, v_tok, kc, vc, slots)
    lens = np.array([38, 38], np.int32)
    q = rng.uniform(-1, 1, (2, 8, 64)).astype(np.float32)
    out = oracle.decode(q, kc, vc, bt, lens, 0.3)
    # reference: each sequence's own contiguous history + its own token, by library attention
    for b in range(2):
        K = np.concatenate([widen(case.logical_k[0][:37]), k_tok[b][None]], 0)
        V = np.concatenate([widen(case.logical_v[0][:37]), v_tok[b][None]], 0)
        o = F.scaled_dot_product_attention(torch.from_numpy(q[b].astype(np.float64))[None, :, None, :],
                                           torch.from_numpy(K).permute(1, 0, 2)[None],
                                           torch.from_numpy(V).permute(1, 0, 2)[None], scale=0.3, enable_gqa=True)
        assert np.abs(out[b] - o[0, :, 0, :].numpy()).max() <= TOL


def test_swap_out_and_in_preserves_attention():
    case = small_decode_case(191, dtype="bf16", D=128)
    kc, vc = written(case)
    base = oracle.decode(case.q, kc, vc, case.block_tables, case.context_lens, case.scale)
    used = np.unique(case.block_tables[case.block_tables >= 0])
    host_k = np.zeros((len(used) + 3,) + kc.shape[1:], kc.dtype)
    host_v = np.zeros_like(host_k)
    out_pairs = np.stack([used, np.arange(len(used)) + 3], 1)
    host_k = oracle.swap_blocks(host_k, kc, out_pairs)
    host_v = oracle.swap_blocks(host_v, vc, out_pairs)
    # bring them back to a permuted set of device blocks and rewrite the tables
    new_ids = np.random.default_rng(9).permutation(case.num_blocks)[:len(used)]
    in_pairs = np.stack([np.arange(len(used)) + 3, new_ids], 1)
    kc2 = oracle.swap_blocks(np.full_like(kc, 0), host_k, in_pairs)
    vc2 = oracle.swap_blocks(np.full_like(vc, 0), host_v, in_pairs)
    remap = dict(zip(used.tolist(), new_ids.tolist()))
    bt2 = np.vectorize(lambda x: remap.get(int(x), -1))(case.block_tables).astype(np.int32)
    moved = oracle.decode(case.q, kc2, vc2, bt2, case.context_lens, case.scale)
    assert np.array_equal(base, moved)


def test_block_copy_rejects_indices_outside_the_pool():
    case = small_decode_case(201)
    with pytest.raises(oracle.OracleError):
        oracle.copy_blocks(case.k_cache, case.v_cache, [[0, case.num_blocks]])


def test_varlen_batch_matches_library_per_sequence():
    # one batch mixing a sequence with no new tokens, decode tokens, verify chunks and a
    # long chunk (the shape a continuous-batching step hands to one launch): every row
    # equals the library's masked attention for its own sequence, whatever its neighbours
    case = W.make_case("pin_varlen", 171, context_lens=[9, 40, 3, 130, 77, 200, 1], q_lens=[0, 1, 3, 4, 77, 37, 1],
                       num_heads=8, num_kv_heads=2, head_dim=64, dtype="f32", scale=0.29, keep_logical=True,
                       table_slack=1)
    kc, vc = written(case)
    got = oracle.prefill(case.q, kc, vc, case.block_tables, case.cu_q_lens, case.context_lens, case.scale)
    ref = sdpa_prefill(case)
    assert got.shape == ref.shape == (int(case.q_lens.sum()), 8, 64)
    assert np.abs(got - ref).max() <= 1e-12
