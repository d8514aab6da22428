"""GPU parity of the tcgen05 chunked-prefill kernel against the fp64 oracle.

Each case writes the step's tokens with pa_reshape_and_cache, then runs
pa_prefill_chunk over every sequence's chunk (causal, at its context offset),
all through the C ABI. bf16 outputs must be within 5e-3 max abs error of the
oracle on every compared element.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_366_b200 import workloads as W
from gpu_util import TOL, DevCase, max_err, mixed_step_reference, oracle_written, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_366_b200 import pa as _pa
    assert _pa.pa_get_status() == 0
    return _pa


def run_prefill(pa, case, seqs=None):
    d = DevCase(case)
    pa.pa_reshape_and_cache(d.k_new, d.v_new, d.k_cache, d.v_cache, d.slot_mapping)
    seqs = np.arange(case.num_seqs) if seqs is None else np.asarray(seqs)
    s0, s1 = int(seqs[0]), int(seqs[-1]) + 1
    r0, r1 = int(case.cu_q_lens[s0]), int(case.cu_q_lens[s1])
    q = d.q[r0:r1].contiguous()
    out = torch.full_like(q, float("nan"))
    cu = (d.cu_q_lens[s0:s1 + 1] - r0).contiguous()
    max_q = int(case.q_lens[s0:s1].max())
    pa.pa_prefill_chunk(out, q, d.k_cache, d.v_cache, d.block_tables[s0:s1], cu, d.context_lens[s0:s1], max_q,
                        case.scale)
    status = pa.pa_get_status()
    return out, status, (r0, r1)


def check_prefill(pa, case, seqs=None, rows=None):
    out, status, (r0, r1) = run_prefill(pa, case, seqs)
    assert status == 0, hex(status)
    kc, vc = oracle_written(case)
    seqs = np.arange(case.num_seqs) if seqs is None else np.asarray(seqs)
    s0, s1 = int(seqs[0]), int(seqs[-1]) + 1
    cu = case.cu_q_lens[s0:s1 + 1] - r0
    ref = oracle.prefill(case.q[r0:r1], kc, vc, case.block_tables[s0:s1], cu, case.context_lens[s0:s1],
                         case.scale, rows=rows)
    got = to_host(out)
    if rows is not None:
        got = got[np.asarray(rows)]
    err = max_err(got, ref)
    assert err <= TOL["bf16"], (case.name, err)
    return err


def prefill_case(seed, ctx, ql, H=32, Hk=8, **kw):
    return W.make_case("prefill", seed, context_lens=list(ctx), q_lens=list(ql), num_heads=H, num_kv_heads=Hk,
                       head_dim=128, dtype="bf16", **kw)


def test_single_chunk_offset_zero(pa):
    check_prefill(pa, prefill_case(31, [40], [40]))


@pytest.mark.parametrize("H,Hk", [(32, 8), (8, 8), (16, 8), (64, 8)])
def test_ragged_chunks_at_offsets(pa, H, Hk):
    # chunks cross 16-token blocks, 128-key tiles and the per-CTA token tiles; one starts at offset 0
    case = prefill_case(40 + H, [300, 77, 1000, 129, 16, 513], [77, 77, 129, 1, 16, 200], H=H, Hk=Hk, table_slack=1)
    check_prefill(pa, case)


def test_single_token_chunks_equal_decode(pa):
    case = prefill_case(51, [1, 15, 16, 17, 200, 700, 2049], [1] * 7)
    out, status, _ = run_prefill(pa, case)
    assert status == 0
    d = DevCase(case)
    pa.pa_reshape_and_cache(d.k_new, d.v_new, d.k_cache, d.v_cache, d.slot_mapping)
    dec = torch.empty_like(d.q)
    shape = pa.shape_of(d.k_cache, case.num_heads)
    ws = torch.empty(max(16, pa.pa_decode_workspace_bytes(7, 2049, 0, shape)), dtype=torch.uint8, device="cuda")
    pa.pa_decode(dec, d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, 2049, case.scale, 0, ws)
    assert pa.pa_get_status() == 0
    diff = (out.float() - dec.float()).abs().max().item()
    assert diff <= 2 * TOL["bf16"], diff
    check_prefill(pa, case)


def test_long_chunk_two_sequences(pa):
    case = prefill_case(61, [2500, 1800], [700, 1800])
    check_prefill(pa, case)


def test_mixed_step_prefill_every_row(pa):
    # the mixed step's 2048-token chunk at offset 6144 (64 K/V tiles per Q tile), all 2048 x 32 x 128
    # outputs against the oracle
    case, ref = mixed_step_reference()
    out, status, (r0, r1) = run_prefill(pa, case, seqs=[0])
    assert status == 0, hex(status)
    assert (r0, r1) == (0, 2048)
    err = max_err(to_host(out), ref[r0:r1])
    assert err <= TOL["bf16"], err


def test_bad_chunk_lengths_flag_status(pa):
    case = prefill_case(71, [64, 64], [16, 16])
    d = DevCase(case)
    out = torch.empty_like(d.q)
    cu = d.cu_q_lens.clone()
    lens = d.context_lens.clone()
    lens[1] = 3  # shorter than its chunk of 16
    pa.pa_prefill_chunk(out, d.q, d.k_cache, d.v_cache, d.block_tables, cu, lens, 16, case.scale)
    assert pa.pa_get_status() & pa.PA_STATUS_BAD_QUERY
