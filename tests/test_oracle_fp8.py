"""Pins for the oracle's FP8 E4M3 codec and FP8-cache attention (CPU).

E4M3 ("fn"): 1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no
infinities, S.1111.111 is NaN, largest finite 448, subnormals k * 2^-9. The
codes below are worked out by hand from that definition. torch's
float8_e4m3fn conversion (a library routine) is a second pin over the finite
range. FP8-cache attention must equal plain attention over the dequantized
cache.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_366_b200 import workloads as W

# (value, code): exact values, round-to-nearest-even ties, the subnormal range and saturation
GOLDEN = [
    (1.0, 0x38), (-2.0, 0xC0), (0.5, 0x30), (448.0, 0x7E), (-448.0, 0xFE), (2.0 ** -6, 0x08), (2.0 ** -9, 0x01),
    (7 * 2.0 ** -9, 0x07), (1.125, 0x39), (1.0625, 0x38), (1.1875, 0x3A), (2.0 ** -10, 0x00),
    (3 * 2.0 ** -11, 0x01), (464.0, 0x7E), (500.0, 0x7E), (1e9, 0x7E), (-0.0, 0x80), (0.0, 0x00),
    (240.0, 0x77), (256.0, 0x78), (272.0, 0x78), (288.0, 0x79),
]


@pytest.mark.parametrize("value,code", GOLDEN)
def test_e4m3_golden_codes(value, code):
    assert oracle.e4m3_encode(value) == code, hex(oracle.e4m3_encode(value))


def test_e4m3_every_code_round_trips():
    for c in range(256):
        v = oracle.e4m3_decode(c)
        if c in (0x7F, 0xFF):
            assert np.isnan(v)
        else:
            assert oracle.e4m3_encode(v) == c


def test_e4m3_decode_values():
    assert oracle.e4m3_decode(0x7E) == 448.0 and oracle.e4m3_decode(0x01) == 2.0 ** -9
    assert oracle.e4m3_decode(0x3F) == 1.875 and oracle.e4m3_decode(0xB8) == -1.0


def test_e4m3_matches_torch_in_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-448, 448, 4000), rng.uniform(-0.05, 0.05, 4000),
                        rng.uniform(-2.0 ** -6, 2.0 ** -6, 2000)]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(v) for v in x], np.uint8)
    assert np.array_equal(got, ref)


def _fp8_pool(case, k_scale, v_scale):
    """Quantize a bf16 case's whole pool (used slots) to E4M3 codes with the oracle's write."""
    NB, bs, Hk, D = case.k_cache.shape
    slots = np.arange(NB * bs, dtype=np.int64)
    rows_k = case.k_cache.reshape(NB * bs, Hk, D)
    rows_v = case.v_cache.reshape(NB * bs, Hk, D)
    zk = np.zeros((NB, bs, Hk, D), np.uint8)
    kc, vc = oracle.reshape_and_cache_fp8(rows_k, rows_v, zk, zk.copy(), slots, np.float32(1) / np.float32(k_scale),
                                          np.float32(1) / np.float32(v_scale))
    return kc, vc


def test_fp8_decode_equals_attention_over_dequantized_cache():
    case = W.make_case("fp8", 221, context_lens=[1, 37, 100, 300], q_lens=[1] * 4, num_heads=8, num_kv_heads=2,
                       head_dim=64, dtype="bf16")
    kc_bf, vc_bf = oracle.reshape_and_cache(case.k_new, case.v_new, case.k_cache, case.v_cache, case.slot_mapping)
    case.k_cache, case.v_cache = kc_bf, vc_bf
    ks, vs = 0.5, 0.25  # powers of two: dequantized values are exact in fp32
    kc, vc = _fp8_pool(case, ks, vs)
    got = oracle.decode_fp8(case.q, kc, vc, ks, vs, case.block_tables, case.context_lens, case.scale)
    deq = np.vectorize(oracle.e4m3_decode)
    kf = (deq(kc) * ks).astype(np.float32)
    vf = (deq(vc) * vs).astype(np.float32)
    qf = W.bf16_bits_to_f32(case.q)
    ref = oracle.decode(qf, kf, vf, case.block_tables, case.context_lens, case.scale)
    assert np.array_equal(got, ref)


def test_fp8_prefill_equals_attention_over_dequantized_cache():
    # ragged chunks at offsets (one of them a single decode token, one a whole prompt)
    case = W.make_case("fp8p", 222, context_lens=[40, 37, 100, 300], q_lens=[40, 1, 23, 70], num_heads=8,
                       num_kv_heads=2, head_dim=64, dtype="bf16")
    kc_bf, vc_bf = oracle.reshape_and_cache(case.k_new, case.v_new, case.k_cache, case.v_cache, case.slot_mapping)
    case.k_cache, case.v_cache = kc_bf, vc_bf
    ks, vs = 0.5, 0.25  # powers of two: dequantized values are exact in fp32
    kc, vc = _fp8_pool(case, ks, vs)
    got = oracle.prefill_fp8(case.q, kc, vc, ks, vs, case.block_tables, case.cu_q_lens, case.context_lens,
                             case.scale)
    deq = np.vectorize(oracle.e4m3_decode)
    kf = (deq(kc) * ks).astype(np.float32)
    vf = (deq(vc) * vs).astype(np.float32)
    qf = W.bf16_bits_to_f32(case.q)
    ref = oracle.prefill(qf, kf, vf, case.block_tables, case.cu_q_lens, case.context_lens, case.scale)
    assert np.isfinite(ref).all() and np.array_equal(got, ref)
    # the scales are not interchangeable: K's scale sharpens the softmax, V's scales the output
    swapped = oracle.prefill_fp8(case.q, kc, vc, vs, ks, case.block_tables, case.cu_q_lens, case.context_lens,
                                 case.scale)
    assert not np.allclose(swapped, got)
    # a subset of rows gives the same rows
    rows = np.array([0, 39, 40, 41, 63, 64, 133], np.int32)
    sub = oracle.prefill_fp8(case.q, kc, vc, ks, vs, case.block_tables, case.cu_q_lens, case.context_lens,
                             case.scale, rows=rows)
    assert np.array_equal(sub, got[rows])


def test_fp8_prefill_of_single_tokens_equals_fp8_decode():
    case = W.make_case("fp8p1", 223, context_lens=[1, 16, 17, 250], q_lens=[1] * 4, num_heads=8, num_kv_heads=2,
                       head_dim=64, dtype="bf16")
    kc_bf, vc_bf = oracle.reshape_and_cache(case.k_new, case.v_new, case.k_cache, case.v_cache, case.slot_mapping)
    case.k_cache, case.v_cache = kc_bf, vc_bf
    ks, vs = 0.02, 1.0 / 48.0
    kc, vc = _fp8_pool(case, ks, vs)
    dec = oracle.decode_fp8(case.q, kc, vc, ks, vs, case.block_tables, case.context_lens, case.scale)
    pre = oracle.prefill_fp8(case.q, kc, vc, ks, vs, case.block_tables, case.cu_q_lens, case.context_lens,
                             case.scale)
    assert np.isfinite(dec).all() and np.array_equal(pre, dec)


def test_fp8_write_quantizes_in_fp32_then_rounds():
    k = W.f32_to_bf16_bits(np.array([[[0.3, -0.77, 1.0, 0.0]]], np.float32))
    kc = np.zeros((2, 16, 1, 4), np.uint8)
    inv = np.float32(1) / np.float32(0.013)
    out, _ = oracle.reshape_and_cache_fp8(k, k, kc, kc.copy(), np.array([5], np.int64), inv, inv)
    expect = [oracle.e4m3_encode(np.float32(W.bf16_bits_to_f32(k)[0, 0, i]) * inv) for i in range(4)]
    assert list(out[0, 5, 0]) == expect and np.count_nonzero(out) == 3
