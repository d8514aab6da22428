"""GPU parity of one varlen launch over a mixed batch against the fp64 oracle.

A continuous-batching step mixes decode tokens (chunks of 1), short verify
chunks (a few tokens per sequence, the speculative-decoding shape) and long
prefill chunks. pa_prefill_chunk takes all of them in one launch through
cu_q_lens. A CTA whose sequence fills only one Q tile runs its second slot
over the odd K/V tiles and merges the two partial softmaxes, so these tests
cover chunks that end just before, at and just after the 128-key tile edges.
bf16 outputs must be within 5e-3 max abs error of the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_366_b200 import workloads as W
from gpu_util import TOL, DevCase, max_err, mixed_step_reference, oracle_written, to_host, widen

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_366_b200 import pa as _pa
    assert _pa.pa_get_status() == 0
    return _pa


def one_launch(pa, case):
    """Write the step's tokens, then attend every sequence's chunk in a single launch."""
    d = DevCase(case)
    pa.pa_reshape_and_cache(d.k_new, d.v_new, d.k_cache, d.v_cache, d.slot_mapping)
    out = torch.full_like(d.q, float("nan"))
    pa.pa_prefill_chunk(out, d.q, d.k_cache, d.v_cache, d.block_tables, d.cu_q_lens, d.context_lens,
                        int(case.q_lens.max()), case.scale)
    assert pa.pa_get_status() == 0
    return to_host(out)


def check(pa, case, rows=None):
    got = one_launch(pa, case)
    kc, vc = oracle_written(case)
    ref = oracle.prefill(case.q, kc, vc, case.block_tables, case.cu_q_lens, case.context_lens, case.scale,
                         rows=rows)
    if rows is not None:
        got = got[np.asarray(rows)]
    err = max_err(got, ref)
    assert err <= TOL["bf16"], (case.name, err)
    return err


def mixed_case(seed, ctx, ql, H=32, Hk=8):
    return W.make_case("varlen", seed, context_lens=list(ctx), q_lens=list(ql), num_heads=H, num_kv_heads=Hk,
                       head_dim=128, dtype="bf16")


@pytest.mark.parametrize("H,Hk", [(32, 8), (8, 8), (16, 8), (64, 8)])
def test_verify_chunks_at_tile_edges(pa, H, Hk):
    # one Q tile per CTA throughout; contexts of 1, 2 and 3+ key tiles, on and next to the edges
    ctx = [1, 4, 127, 128, 129, 130, 255, 256, 257, 383, 384, 385, 1000, 2049]
    ql = [1, 4, 1, 4, 1, 2, 8, 3, 1, 5, 7, 2, 6, 4]
    check(pa, mixed_case(60 + H, ctx, ql, H=H, Hk=Hk))


def test_verify_chunks_ragged(pa):
    rng = np.random.default_rng(61)
    ql = rng.integers(1, 9, size=40)
    ctx = [int(rng.integers(q, 3000)) for q in ql]
    check(pa, mixed_case(62, ctx, ql))


def test_decode_prefill_and_verify_in_one_launch(pa):
    # a long chunk in the middle of decode tokens and verify chunks, and one sequence with no tokens
    ctx = [700, 33, 1500, 2600, 900, 129, 5000, 64, 260, 1200, 1800]
    ql = [1, 1, 4, 1000, 0, 1, 1, 7, 200, 1, 3]
    check(pa, mixed_case(63, ctx, ql))


def test_one_launch_matches_pa_decode(pa):
    # decode tokens through the varlen launch and through pa_decode give the same attention
    case = mixed_case(64, [17, 130, 600, 2100, 4097], [1] * 5)
    got = one_launch(pa, case)
    d = DevCase(case)
    pa.pa_reshape_and_cache(d.k_new, d.v_new, d.k_cache, d.v_cache, d.slot_mapping)
    ws = torch.empty(pa.pa_decode_workspace_bytes(case.num_seqs, int(case.context_lens.max()), 0,
                                                  pa.shape_of(d.k_cache, case.num_heads)) + 16,
                     dtype=torch.uint8, device="cuda")
    out = torch.empty_like(d.q)
    pa.pa_decode(out, d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, int(case.context_lens.max()),
                 case.scale, 0, ws)
    assert max_err(got, widen(to_host(out))) <= 2 * TOL["bf16"]


def test_spec_verify_full_size(pa):
    # 64 sequences x 4 tokens at decode-batch lengths: every row
    check(pa, W.spec_verify())


def test_mixed_step_in_one_launch_full_size(pa):
    # the mixed step (2048-token chunk + 192 decode tokens) as one launch: every one of the 2240 rows
    case, ref = mixed_step_reference()
    got = one_launch(pa, case)
    err = max_err(got, ref)
    assert err <= TOL["bf16"], err
