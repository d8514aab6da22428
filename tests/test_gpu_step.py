"""GPU checks of DecodeStep, the end-to-end API (host inputs -> write + decode -> host output).

Both input modes (staged views in one pinned buffer; the caller's own pinned
tensors), with and without CUDA-graph replay, must give the oracle's decode,
and a later step must see the inputs written for it.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_366_b200 import workloads as W
from gpu_util import TOL, max_err, oracle_written

pytestmark = pytest.mark.gpu


def _dev(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _pinned(a):
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if a.dtype == np.uint16 else np.ascontiguousarray(a))
    t = t.pin_memory()
    return t.view(torch.bfloat16) if a.dtype == np.uint16 else t


def _fill(dst, a):
    a = np.ascontiguousarray(a)
    src = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
    (dst.view(torch.int16) if a.dtype == np.uint16 else dst).copy_(src)


def _host_bits(t):
    return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()


def _case(seed):
    return W.make_case("step", seed, context_lens=[5, 130, 700, 1500], q_lens=[1] * 4, num_heads=32,
                       num_kv_heads=8, head_dim=128, dtype="bf16")


def _reference(case):
    kc, vc = oracle_written(case)
    return oracle.decode(case.q, kc, vc, case.block_tables, case.context_lens, case.scale)


@pytest.mark.parametrize("staged", [True, False])
@pytest.mark.parametrize("use_graph", [True, False])
def test_decode_step_matches_oracle(staged, use_graph):
    from paged_kv_cache_366_b200.step import DecodeStep
    case = _case(70)
    step = DecodeStep(_dev(case.k_cache), _dev(case.v_cache), case.num_heads, case.num_seqs,
                      case.max_blocks_per_seq, int(case.context_lens.max()), case.scale, use_graph=use_graph)
    names = ["q", "k_new", "v_new", "slot_mapping", "block_tables", "context_lens"]
    arrays = [case.q, case.k_new, case.v_new, case.slot_mapping, case.block_tables, case.context_lens]
    if staged:
        views = step.inputs()
        for n, a in zip(names, arrays):
            _fill(views[n], a)
    else:
        out_h = torch.empty((case.num_seqs, case.num_heads, case.head_dim), dtype=torch.int16).pin_memory()
        step.bind(*[_pinned(a) for a in arrays], out_h.view(torch.bfloat16))
    got = _host_bits(step.run())
    assert max_err(got, _reference(case)) <= TOL["bf16"]
    # a second step with new queries written into the same host buffers
    q2 = W.f32_to_bf16_bits(-W.bf16_bits_to_f32(case.q))
    if staged:
        _fill(views["q"], q2)
    else:
        step._host[0].view(torch.int16).copy_(torch.from_numpy(q2.view(np.int16)))
    got2 = _host_bits(step.run())
    case.q = q2
    assert max_err(got2, _reference(case)) <= TOL["bf16"]
    assert step.h2d_bytes() >= sum(a.nbytes for a in arrays)
