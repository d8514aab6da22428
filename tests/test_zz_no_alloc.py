"""pa_decode_noalloc: the decode entry point for callers that cannot allocate.

Some callers cannot get device memory for a workspace: a graph being captured
in a mode that forbids allocation, an engine that owns all of HBM, plugin code
without access to the host's allocator. pa_decode_noalloc serves them by
putting the split-context partials in a scratch array built into the library.
This checks, through the C ABI, that it returns what pa_decode returns with a
caller-allocated workspace. It does so on two calls in a row, the second on
different sequences, so the second call starts with the first call's leftovers
in the shared array. It also checks that a request too big for the array is
refused before anything is launched.

This file sorts last so that a run stopping at the first failure has already
run every other test. It also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_366_b200 import workloads as W
from gpu_util import TOL, DevCase, to_host, widen

pytestmark = pytest.mark.gpu


def _with_workspace(pa, d, case, max_ctx, part):
    out = torch.full_like(d.q, float("nan"))
    n = pa.pa_decode_workspace_bytes(case.num_seqs, max_ctx, part, pa.shape_of(d.k_cache, case.num_heads))
    ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
    pa.pa_decode(out, d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, max_ctx, case.scale, part, ws)
    return out


def test_noalloc_matches_decode_on_two_calls_in_a_row():
    assert torch.cuda.is_available()
    from paged_kv_cache_366_b200 import pa

    cases = [
        W.make_case("noalloc_a", 21, context_lens=[6000, 17, 3000, 512, 4097, 1, 2500, 800], q_lens=[1] * 8,
                    num_heads=32, num_kv_heads=8, head_dim=128, dtype="bf16"),
        W.make_case("noalloc_b", 22, context_lens=[1500, 3333, 64, 2049, 700], q_lens=[1] * 5, num_heads=32,
                    num_kv_heads=8, head_dim=128, dtype="bf16"),
    ]
    for case in cases:
        d = DevCase(case)
        pa.pa_reshape_and_cache(d.k_new, d.v_new, d.k_cache, d.v_cache, d.slot_mapping)
        max_ctx = int(case.context_lens.max())
        shape = pa.shape_of(d.k_cache, case.num_heads)
        part = 256
        need = pa.pa_decode_workspace_bytes(case.num_seqs, max_ctx, part, shape)
        assert 0 < need <= pa.PA_NOALLOC_SCRATCH_BYTES  # the split-context path really uses the scratch
        ref = _with_workspace(pa, d, case, max_ctx, part)
        got = torch.full_like(d.q, float("nan"))
        pa.pa_decode_noalloc(got, d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, max_ctx, case.scale,
                             part)
        assert pa.pa_get_status() == 0
        err = float(np.abs(widen(to_host(got)) - widen(to_host(ref))).max())
        assert np.isfinite(err) and err <= TOL[case.dtype], (case.name, err)


def test_noalloc_refuses_requests_beyond_its_scratch():
    from paged_kv_cache_366_b200 import pa

    case = W.make_case("noalloc_big", 23, context_lens=[64, 64], q_lens=[1, 1], num_heads=32, num_kv_heads=8,
                       head_dim=128, dtype="bf16")
    d = DevCase(case)
    shape = pa.shape_of(d.k_cache, case.num_heads)
    # 2 sequences x 32 heads x P partitions x (128 + 2) floats > 16 MiB for P > 504
    huge = 64 * 600
    assert pa.pa_decode_workspace_bytes(2, huge, 64, shape) > pa.PA_NOALLOC_SCRATCH_BYTES
    out = torch.empty_like(d.q)
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode_noalloc(out, d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, huge, case.scale, 64)
    assert e.value.code == pa.PA_ERR_SCRATCH_LIMIT
    assert pa.pa_get_status() == 0
