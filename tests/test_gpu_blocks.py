"""GPU parity of the whole-block copies (copy-on-write fork, swap out/in) against the oracle.

Copies must be bit-exact. The fork and swap scenarios then decode through the
C ABI and compare with the fp64 oracle within the attention tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_366_b200 import workloads as W
from gpu_util import TOL, DevCase, max_err, oracle_written, to_dev, to_host, decode_workspace

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_366_b200 import pa as _pa
    assert _pa.pa_get_status() == 0
    return _pa


def test_copy_blocks_bit_exact(pa):
    case = W.decode_batch()
    d = DevCase(case)
    rng = np.random.default_rng(5)
    used = np.unique(case.block_tables[case.block_tables >= 0])
    free = np.setdiff1d(np.arange(case.num_blocks), used)
    n = 700
    pairs = np.stack([rng.choice(used, n), rng.choice(free, n, replace=False)], 1).astype(np.int64)
    pa.pa_copy_blocks(d.k_cache, d.v_cache, to_dev(pairs))
    assert pa.pa_get_status() == 0
    kc, vc = oracle.copy_blocks(case.k_cache, case.v_cache, pairs)
    assert np.array_equal(to_host(d.k_cache).view(np.uint16), kc)
    assert np.array_equal(to_host(d.v_cache).view(np.uint16), vc)


def test_copy_on_write_fork_then_decode(pa):
    case = W.make_case("fork", 181, context_lens=[37, 37], q_lens=[0, 0], num_heads=32, num_kv_heads=8,
                       head_dim=128, dtype="bf16", shared_prefix_blocks=2, table_slack=1)
    bt = case.block_tables.copy()
    bt[1, :3] = bt[0, :3]
    free = np.setdiff1d(np.arange(case.num_blocks), bt[bt >= 0])
    pairs = np.array([[bt[0, 2], free[0]]], np.int64)
    bt[1, 2] = free[0]
    rng = np.random.default_rng(3)
    k_tok = W.f32_to_bf16_bits(rng.uniform(-1, 1, (2, 8, 128)).astype(np.float32))
    v_tok = W.f32_to_bf16_bits(rng.uniform(-1, 1, (2, 8, 128)).astype(np.float32))
    q = W.f32_to_bf16_bits(rng.uniform(-1, 1, (2, 32, 128)).astype(np.float32))
    slots = np.array([oracle.slot_of(bt[0], 37), oracle.slot_of(bt[1], 37)], np.int64)
    lens = np.array([38, 38], np.int32)

    d = DevCase(case)
    pa.pa_copy_blocks(d.k_cache, d.v_cache, to_dev(pairs))
    pa.pa_reshape_and_cache(to_dev(k_tok), to_dev(v_tok), d.k_cache, d.v_cache, to_dev(slots))
    out = torch.empty((2, 32, 128), dtype=torch.bfloat16, device="cuda")
    pa.pa_decode(out, to_dev(q), d.k_cache, d.v_cache, to_dev(bt), to_dev(lens), 38, case.scale, 0,
                 decode_workspace(pa, 2, 38, d.k_cache, 32))
    assert pa.pa_get_status() == 0

    kc, vc = oracle.copy_blocks(case.k_cache, case.v_cache, pairs)
    kc, vc = oracle.reshape_and_cache(k_tok, v_tok, kc, vc, slots)
    ref = oracle.decode(q, kc, vc, bt, lens, case.scale)
    assert max_err(to_host(out), ref) <= TOL["bf16"]
    # the two sequences now differ only in their last token, so their outputs differ
    assert not torch.equal(out[0], out[1])


def test_swap_out_to_pinned_host_and_back(pa):
    case = W.make_case("swap", 211, context_lens=[300, 1000, 77, 2049], q_lens=[1] * 4, num_heads=32,
                       num_kv_heads=8, head_dim=128, dtype="bf16")
    d = DevCase(case)
    pa.pa_reshape_and_cache(d.k_new, d.v_new, d.k_cache, d.v_cache, d.slot_mapping)
    used = np.unique(case.block_tables[case.block_tables >= 0])
    n = len(used)
    host_k = torch.zeros((n + 5,) + tuple(d.k_cache.shape[1:]), dtype=torch.bfloat16).pin_memory()
    host_v = torch.zeros_like(host_k).pin_memory()
    out_pairs = torch.from_numpy(np.stack([used, np.arange(n) + 5], 1).astype(np.int64)).pin_memory()
    pa.pa_swap_blocks(host_k, d.k_cache, out_pairs)
    pa.pa_swap_blocks(host_v, d.v_cache, out_pairs)
    torch.cuda.synchronize()
    assert pa.pa_get_status() == 0
    kc_ref, vc_ref = oracle_written(case)
    assert np.array_equal(host_k.view(torch.int16).numpy().view(np.uint16)[5:], kc_ref[used])
    # swap back in to a permuted set of blocks of a fresh pool, rewrite the tables, decode
    new_ids = np.random.default_rng(9).permutation(case.num_blocks)[:n]
    in_pairs = to_dev(np.stack([np.arange(n) + 5, new_ids], 1).astype(np.int64))
    kc2 = torch.zeros_like(d.k_cache)
    vc2 = torch.zeros_like(d.v_cache)
    pa.pa_swap_blocks(kc2, host_k, in_pairs)
    pa.pa_swap_blocks(vc2, host_v, in_pairs)
    remap = dict(zip(used.tolist(), new_ids.tolist()))
    bt2 = np.vectorize(lambda x: remap.get(int(x), -1))(case.block_tables).astype(np.int32)
    out = torch.empty_like(d.q)
    ws = torch.empty(max(16, pa.pa_decode_workspace_bytes(4, 2049, 0, pa.shape_of(kc2, 32))), dtype=torch.uint8,
                     device="cuda")
    pa.pa_decode(out, d.q, kc2, vc2, to_dev(bt2), d.context_lens, 2049, case.scale, 0, ws)
    assert pa.pa_get_status() == 0
    ref = oracle.decode(case.q, kc_ref, vc_ref, case.block_tables, case.context_lens, case.scale)
    assert max_err(to_host(out), ref) <= TOL["bf16"]


def test_swap_refuses_pageable_host_memory(pa):
    src = torch.zeros((4, 16, 8, 128), dtype=torch.bfloat16, device="cuda")
    dst = torch.zeros((4, 16, 8, 128), dtype=torch.bfloat16)  # not pinned
    pairs = torch.tensor([[0, 1]], dtype=torch.int64, device="cuda")
    rc = pa.lib.pa_swap_blocks(pa.ctypes.c_void_p(dst.data_ptr()), pa.ctypes.c_void_p(src.data_ptr()),
                               pa.ctypes.c_void_p(pairs.data_ptr()), 1, 4, 4, 16 * 8 * 128 * 2, None)
    assert rc == -1


def test_bad_copy_pair_sets_status(pa):
    k = torch.zeros((8, 16, 2, 64), dtype=torch.float32, device="cuda")
    v = torch.zeros_like(k)
    pa.pa_copy_blocks(k, v, torch.tensor([[0, 8]], dtype=torch.int64, device="cuda"))
    assert pa.pa_get_status() & pa.PA_STATUS_BAD_BLOCK_ID
