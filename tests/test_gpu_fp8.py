"""GPU parity of the FP8 (E4M3) KV cache against the oracle.

The write quantizes bf16 K/V rows into E4M3 codes: it must be bit-exact with
the oracle's quantization (the same fp32 product, then nearest code, ties to
even, saturating). Decode and chunked prefill over an FP8 pool must match the
oracle's decode and prefill over the same codes (dequantized exactly, times the
scales) within 5e-3.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_366_b200 import workloads as W
from gpu_util import TOL, max_err, to_dev, to_host

pytestmark = pytest.mark.gpu

K_SCALE, V_SCALE = 0.02, 1.0 / 48.0


@pytest.fixture(scope="module")
def pa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_366_b200 import pa as _pa
    assert _pa.pa_get_status() == 0
    return _pa


def inv(x):
    return np.float32(1) / np.float32(x)


def fp8_pools(case):
    """E4M3 pools of a bf16 case (every slot, NaN poison included), by the oracle."""
    NB, bs, Hk, D = case.k_cache.shape
    slots = np.arange(NB * bs, dtype=np.int64)
    z = np.zeros((NB, bs, Hk, D), np.uint8)
    return oracle.reshape_and_cache_fp8(case.k_cache.reshape(-1, Hk, D), case.v_cache.reshape(-1, Hk, D), z, z.copy(),
                                        slots, inv(K_SCALE), inv(V_SCALE))


def test_fp8_write_bit_exact(pa):
    case = W.decode_batch()
    kc0, vc0 = fp8_pools(case)
    kc, vc = to_dev(kc0), to_dev(vc0)
    pa.pa_reshape_and_cache(to_dev(case.k_new), to_dev(case.v_new), kc, vc, to_dev(case.slot_mapping),
                            k_scale=K_SCALE, v_scale=V_SCALE)
    assert pa.pa_get_status() == 0
    kr, vr = oracle.reshape_and_cache_fp8(case.k_new, case.v_new, kc0, vc0, case.slot_mapping, inv(K_SCALE),
                                          inv(V_SCALE))
    assert np.array_equal(to_host(kc), kr) and np.array_equal(to_host(vc), vr)


def check_fp8_decode(pa, case, partition_tokens=0):
    kc0, vc0 = fp8_pools(case)
    kc, vc = to_dev(kc0), to_dev(vc0)
    pa.pa_reshape_and_cache(to_dev(case.k_new), to_dev(case.v_new), kc, vc, to_dev(case.slot_mapping),
                            k_scale=K_SCALE, v_scale=V_SCALE)
    q = to_dev(case.q)
    out = torch.full_like(q, float("nan"))
    max_ctx = int(case.context_lens.max())
    shape = pa.shape_of(kc, case.num_heads, K_SCALE, V_SCALE)
    n = pa.pa_decode_workspace_bytes(case.num_seqs, max_ctx, partition_tokens, shape)
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
    pa.pa_decode(out, q, kc, vc, to_dev(case.block_tables), to_dev(case.context_lens), max_ctx, case.scale,
                 partition_tokens, ws, k_scale=K_SCALE, v_scale=V_SCALE)
    assert pa.pa_get_status() == 0
    kr, vr = oracle.reshape_and_cache_fp8(case.k_new, case.v_new, kc0, vc0, case.slot_mapping, inv(K_SCALE),
                                          inv(V_SCALE))
    ref = oracle.decode_fp8(case.q, kr, vr, K_SCALE, V_SCALE, case.block_tables, case.context_lens, case.scale)
    err = max_err(to_host(out), ref)
    assert err <= TOL["bf16"], err


def test_fp8_decode_batch(pa):
    check_fp8_decode(pa, W.decode_batch())


@pytest.mark.parametrize("partition_tokens", [0, 64])
@pytest.mark.parametrize("H,Hk,D", [(32, 8, 128), (16, 2, 64), (8, 8, 128), (64, 8, 128)])
def test_fp8_ragged(pa, H, Hk, D, partition_tokens):
    ctx = [1, 15, 16, 17, 64, 65, 200, 1031]
    case = W.make_case("fp8r", 3 + H, context_lens=ctx, q_lens=[1] * len(ctx), num_heads=H, num_kv_heads=Hk,
                       head_dim=D, dtype="bf16", table_slack=1)
    check_fp8_decode(pa, case, partition_tokens)


@pytest.mark.parametrize("H,Hk", [(32, 8), (64, 8)])
def test_fp8_long_ragged_list(pa, H, Hk):
    # units of 1 to 1250 blocks spread over every CTA: the merge runs four warps per unit
    ctx = [1, 2, 17, 20000, 9000, 3000, 15, 16384, 100, 4097]
    case = W.make_case("fp8long", 80 + H, context_lens=ctx, q_lens=[1] * len(ctx), num_heads=H, num_kv_heads=Hk,
                       head_dim=128, dtype="bf16")
    check_fp8_decode(pa, case)


def check_fp8_prefill(pa, case):
    """Every row of every chunk through pa_prefill_chunk over an FP8 pool, against the oracle's FP8 prefill
    over the same codes."""
    kc0, vc0 = fp8_pools(case)
    kc, vc = to_dev(kc0), to_dev(vc0)
    pa.pa_reshape_and_cache(to_dev(case.k_new), to_dev(case.v_new), kc, vc, to_dev(case.slot_mapping),
                            k_scale=K_SCALE, v_scale=V_SCALE)
    q = to_dev(case.q)
    out = torch.full_like(q, float("nan"))
    pa.pa_prefill_chunk(out, q, kc, vc, to_dev(case.block_tables), to_dev(case.cu_q_lens),
                        to_dev(case.context_lens), int(case.q_lens.max()), case.scale, k_scale=K_SCALE,
                        v_scale=V_SCALE)
    assert pa.pa_get_status() == 0
    kr, vr = oracle.reshape_and_cache_fp8(case.k_new, case.v_new, kc0, vc0, case.slot_mapping, inv(K_SCALE),
                                          inv(V_SCALE))
    assert np.array_equal(to_host(kc), kr) and np.array_equal(to_host(vc), vr)
    ref = oracle.prefill_fp8(case.q, kr, vr, K_SCALE, V_SCALE, case.block_tables, case.cu_q_lens,
                             case.context_lens, case.scale)
    err = max_err(to_host(out), ref)
    assert err <= TOL["bf16"], (case.name, err)
    return to_host(out)


@pytest.mark.parametrize("H,Hk", [(32, 8), (8, 8), (16, 8), (64, 8)])
def test_fp8_prefill_ragged_chunks(pa, H, Hk):
    # chunks across 16-token blocks, 128-key tiles and per-CTA token tiles; a decode token; one at offset 0
    case = W.make_case("fp8pre", 90 + H, context_lens=[300, 77, 1000, 129, 16, 513, 40],
                       q_lens=[77, 77, 129, 1, 16, 200, 40], num_heads=H, num_kv_heads=Hk, head_dim=128,
                       dtype="bf16", table_slack=1)
    check_fp8_prefill(pa, case)


def test_fp8_prefill_long_chunks(pa):
    # 1800 tokens at offset 0 (both Q tiles of each CTA, 15 K/V tiles) and 700 at offset 1800
    case = W.make_case("fp8long_pre", 97, context_lens=[2500, 1800], q_lens=[700, 1800], num_heads=32,
                       num_kv_heads=8, head_dim=128, dtype="bf16")
    check_fp8_prefill(pa, case)


def test_fp8_decode_tokens_verify_and_prefill_in_one_launch(pa):
    # decode tokens (chunks of 1, split over two S/O slots), verify chunks of 4 and a prefill chunk in
    # one varlen launch
    ctx = [1, 17, 130, 2049, 64, 260, 900]
    ql = [1, 1, 1, 1, 4, 4, 300]
    case = W.make_case("fp8varlen", 98, context_lens=ctx, q_lens=ql, num_heads=32, num_kv_heads=8, head_dim=128,
                       dtype="bf16")
    check_fp8_prefill(pa, case)


def test_fp8_prefill_rejects_a_bad_scale(pa):
    kc = torch.zeros((4, 16, 8, 128), dtype=torch.uint8, device="cuda")
    q = torch.zeros((2, 32, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(pa.PaError) as e:
        pa.pa_prefill_chunk(torch.empty_like(q), q, kc, kc, torch.zeros((1, 4), dtype=torch.int32, device="cuda"),
                            torch.tensor([0, 2], dtype=torch.int32, device="cuda"),
                            torch.tensor([2], dtype=torch.int32, device="cuda"), 2, 0.1, k_scale=0.0,
                            v_scale=1.0)
    assert e.value.code == -1
