"""GPU parity of the cache write and decode attention against the fp64 oracle.

Every call goes through the C ABI (libpa.so via the ctypes binding). Tolerances:
the cache write must be bit-exact; attention outputs are within 5e-3 (bf16) or
1e-5 (fp32) max abs error of the oracle, over every output element.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_366_b200 import workloads as W
from gpu_util import TOL, DevCase, decode_rows, decode_workspace, max_err, oracle_written, to_dev, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_366_b200 import pa as _pa
    assert _pa.pa_get_status() == 0
    return _pa


def run_step(pa, case, seqs=None, partition_tokens=0, dev=None):
    """Write this step's tokens, then decode `seqs` (default: all). Returns (out, k_cache, v_cache, status)."""
    d = dev or DevCase(case)
    pa.pa_reshape_and_cache(d.k_new, d.v_new, d.k_cache, d.v_cache, d.slot_mapping)
    seqs = np.arange(case.num_seqs) if seqs is None else np.asarray(seqs)
    s0, s1 = int(seqs[0]), int(seqs[-1]) + 1
    assert np.array_equal(seqs, np.arange(s0, s1))
    rows = torch.from_numpy(decode_rows(case, seqs)).cuda()
    q = d.q.index_select(0, rows).contiguous()
    out = torch.full_like(q, float("nan"))
    bt = d.block_tables[s0:s1]
    cl = d.context_lens[s0:s1]
    max_ctx = int(case.context_lens[s0:s1].max())
    shape = pa.shape_of(d.k_cache, case.num_heads)
    nbytes = pa.pa_decode_workspace_bytes(len(seqs), max_ctx, partition_tokens, shape)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device="cuda") if nbytes else None
    pa.pa_decode(out, q, d.k_cache, d.v_cache, bt, cl, max_ctx, case.scale, partition_tokens, ws)
    status = pa.pa_get_status()
    return out, d.k_cache, d.v_cache, status


def check_case(pa, case, seqs=None, partition_tokens=0, check_cache=True):
    out, kc, vc, status = run_step(pa, case, seqs, partition_tokens)
    assert status == 0, hex(status)
    kc_ref, vc_ref = oracle_written(case)
    if check_cache:
        assert np.array_equal(to_host(kc).view(np.uint8), kc_ref.view(np.uint8)), "k_cache write not bit-exact"
        assert np.array_equal(to_host(vc).view(np.uint8), vc_ref.view(np.uint8)), "v_cache write not bit-exact"
    seqs = np.arange(case.num_seqs) if seqs is None else np.asarray(seqs)
    q_np = case.q[decode_rows(case, seqs)]
    ref = oracle.decode(q_np, kc_ref, vc_ref, case.block_tables[seqs], case.context_lens[seqs], case.scale)
    err = max_err(to_host(out), ref)
    assert err <= TOL[case.dtype], (case.name, err)
    return out, err


def test_tiny(pa):
    check_case(pa, W.tiny(keep_logical=False))


@pytest.mark.parametrize("partition_tokens", [0, 64, 192])
@pytest.mark.parametrize("dtype,H,Hk,D", [
    ("bf16", 32, 8, 128), ("bf16", 8, 8, 128), ("bf16", 16, 8, 64), ("bf16", 16, 2, 128),
    ("f32", 8, 2, 64), ("f32", 4, 4, 128), ("f32", 16, 2, 128), ("bf16", 4, 1, 64),
])
def test_ragged_contexts(pa, dtype, H, Hk, D, partition_tokens):
    ctx = [1, 15, 16, 17, 63, 64, 65, 200, 513, 1000, 1031]
    case = W.make_case("ragged", 7 + H + D, context_lens=ctx, q_lens=[1] * len(ctx), num_heads=H, num_kv_heads=Hk,
                       head_dim=D, dtype=dtype, table_slack=2)
    check_case(pa, case, partition_tokens=partition_tokens)


def test_decode_batch_full(pa):
    check_case(pa, W.decode_batch())


def test_long_context_full(pa):
    check_case(pa, W.long_context())


# A long ragged list: units of 1 to 1250 blocks, cut by the automatic slicing over every CTA, so
# that most units are spread over many warps and several CTAs.
LONG_RAGGED_CTX = [1, 2, 17, 20000, 9000, 3000, 15, 16384, 100, 4097]


@pytest.mark.parametrize("dtype,H,Hk,D", [
    ("bf16", 32, 8, 128), ("bf16", 64, 8, 128), ("bf16", 8, 8, 64), ("f32", 32, 8, 128), ("bf16", 16, 8, 128),
    ("f32", 16, 8, 64),
])
def test_long_ragged_list(pa, dtype, H, Hk, D):
    # twice on one workspace of random bytes: the second call starts on the first one's leftovers
    case = W.make_case("long_ragged", 40 + H + D, context_lens=LONG_RAGGED_CTX, q_lens=[1] * len(LONG_RAGGED_CTX),
                       num_heads=H, num_kv_heads=Hk, head_dim=D, dtype=dtype)
    d = DevCase(case)
    pa.pa_reshape_and_cache(d.k_new, d.v_new, d.k_cache, d.v_cache, d.slot_mapping)
    kc_ref, vc_ref = oracle_written(case)
    ref = oracle.decode(case.q, kc_ref, vc_ref, case.block_tables, case.context_lens, case.scale)
    mx = int(case.context_lens.max())
    shape = pa.shape_of(d.k_cache, H)
    g = torch.Generator(device="cuda").manual_seed(9)
    ws = torch.randint(0, 256, (pa.pa_decode_workspace_bytes(case.num_seqs, mx, 0, shape),), dtype=torch.uint8,
                       device="cuda", generator=g)
    for _ in range(2):
        out = torch.full_like(d.q, float("nan"))
        pa.pa_decode(out, d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, mx, case.scale, 0, ws)
        assert pa.pa_get_status() == 0
        err = max_err(to_host(out), ref)
        assert err <= TOL[dtype], err


@pytest.mark.parametrize("partition_tokens", [0, 64])
def test_many_sequences_merge_from_records(pa, partition_tokens):
    # more than 256 sequences: the merge kernel finds each unit's slices in the records the decode
    # kernel wrote (fewer sequences let it compute them from the lengths); units cut at every size
    rng = np.random.default_rng(17)
    ctx = [int(x) for x in rng.integers(1, 700, size=300)]
    case = W.make_case("many", 18, context_lens=ctx, q_lens=[1] * len(ctx), num_heads=16, num_kv_heads=4,
                       head_dim=128, dtype="bf16")
    d = DevCase(case)
    pa.pa_reshape_and_cache(d.k_new, d.v_new, d.k_cache, d.v_cache, d.slot_mapping)
    kc_ref, vc_ref = oracle_written(case)
    ref = oracle.decode(case.q, kc_ref, vc_ref, case.block_tables, case.context_lens, case.scale)
    mx = int(case.context_lens.max())
    n = pa.pa_decode_workspace_bytes(case.num_seqs, mx, partition_tokens, pa.shape_of(d.k_cache, 16))
    ws = torch.full((n,), 255, dtype=torch.uint8, device="cuda")
    out = torch.full_like(d.q, float("nan"))
    pa.pa_decode(out, d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, mx, case.scale, partition_tokens, ws)
    assert pa.pa_get_status() == 0
    assert max_err(to_host(out), ref) <= TOL["bf16"]


@pytest.mark.parametrize("partition_tokens", [128, 192, 320, 512, 1024])
def test_partition_sizes_on_filled_workspace(pa, partition_tokens):
    # slices of 2 to 17 blocks over units of 1 to 65 blocks: units cut at every kind of place,
    # on a workspace of 0xff bytes (NaN if any partial or record were read before it is written)
    ctx = [1, 15, 16, 17, 63, 64, 65, 200, 513, 1000, 1031]
    case = W.make_case("ragged", 7 + 32 + 128, context_lens=ctx, q_lens=[1] * len(ctx), num_heads=32, num_kv_heads=8,
                       head_dim=128, dtype="bf16", table_slack=2)
    d = DevCase(case)
    pa.pa_reshape_and_cache(d.k_new, d.v_new, d.k_cache, d.v_cache, d.slot_mapping)
    kc_ref, vc_ref = oracle_written(case)
    ref = oracle.decode(case.q, kc_ref, vc_ref, case.block_tables, case.context_lens, case.scale)
    mx = int(case.context_lens.max())
    n = pa.pa_decode_workspace_bytes(case.num_seqs, mx, partition_tokens, pa.shape_of(d.k_cache, 32))
    ws = torch.full((n,), 255, dtype=torch.uint8, device="cuda")
    out = torch.full_like(d.q, float("nan"))
    pa.pa_decode(out, d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, mx, case.scale, partition_tokens, ws)
    assert pa.pa_get_status() == 0
    assert max_err(to_host(out), ref) <= TOL["bf16"]


@pytest.mark.parametrize("name,part", [("decode_batch", 0), ("long_context", 0), ("decode_batch", 256)])
def test_partials_then_merge_equals_decode(pa, name, part):
    # pa_decode's two launches called one by one give its output bit for bit
    case = W.CONFIGS[name]()
    d = DevCase(case)
    pa.pa_reshape_and_cache(d.k_new, d.v_new, d.k_cache, d.v_cache, d.slot_mapping)
    mx = int(case.context_lens.max())
    n = pa.pa_decode_workspace_bytes(case.num_seqs, mx, part, pa.shape_of(d.k_cache, case.num_heads))
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    args = (d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, mx, case.scale, part, ws)
    a = torch.full_like(d.q, float("nan"))
    pa.pa_decode(a, *args)
    b = torch.full_like(d.q, float("nan"))
    pa.pa_decode_partials(b, *args)
    pa.pa_decode_merge(b, *args)
    assert pa.pa_get_status() == 0
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_prefix_sharing_shared_equals_copied(pa):
    a = W.prefix_sharing(copy_shared=False)
    out_a, err_a = check_case(pa, a)
    b = W.prefix_sharing(copy_shared=True)
    out_b, _ = check_case(pa, b, check_cache=False)
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16)), "shared-block and copied-block runs differ"


def test_mixed_step_decode_part(pa):
    case = W.mixed_step()
    check_case(pa, case, seqs=np.arange(1, case.num_seqs))


def test_zero_context_gives_zeros(pa):
    case = W.make_case("z", 3, context_lens=[5, 40], q_lens=[1, 1], num_heads=8, num_kv_heads=2, head_dim=128,
                       dtype="bf16")
    d = DevCase(case)
    d.context_lens[0] = 0
    out, _, _, status = run_step(pa, case, dev=d)
    assert status == 0
    o = out.float().cpu().numpy()
    assert np.all(o[0] == 0) and np.all(np.isfinite(o[1]))


def test_decode_is_deterministic(pa):
    case = W.make_case("det", 5, context_lens=[700, 3000, 33], q_lens=[1, 1, 1], num_heads=32, num_kv_heads=8,
                       head_dim=128, dtype="bf16")
    a, *_ = run_step(pa, case)
    b, *_ = run_step(pa, case)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_negative_slot_is_skipped(pa):
    case = W.make_case("neg", 9, context_lens=[20, 30], q_lens=[1, 1], num_heads=8, num_kv_heads=2, head_dim=64,
                       dtype="f32")
    d = DevCase(case)
    d.slot_mapping[0] = -1
    before = d.k_cache.clone()
    pa.pa_reshape_and_cache(d.k_new, d.v_new, d.k_cache, d.v_cache, d.slot_mapping)
    assert pa.pa_get_status() == 0
    changed = (before.view(torch.int32) != d.k_cache.view(torch.int32)).reshape(-1, 2 * 64).any(dim=1)
    rows = torch.nonzero(changed).flatten().cpu().numpy()
    assert list(rows) == [int(case.slot_mapping[1])]


def test_bad_inputs_set_status_not_fault(pa):
    case = W.make_case("bad", 11, context_lens=[40, 90], q_lens=[1, 1], num_heads=8, num_kv_heads=2, head_dim=128,
                       dtype="bf16", table_slack=1)
    d = DevCase(case)
    # slot outside the pool: skipped and flagged
    d.slot_mapping[0] = case.num_blocks * 16 + 3
    pa.pa_reshape_and_cache(d.k_new, d.v_new, d.k_cache, d.v_cache, d.slot_mapping)
    assert pa.pa_get_status() & pa.PA_STATUS_BAD_SLOT
    # a table entry outside the pool in sequence 0: flagged, sequence 1 unaffected
    d.block_tables[0, 1] = case.num_blocks + 5
    out = torch.empty_like(d.q)
    pa.pa_decode(out, d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, 90, case.scale, 0,
                 decode_workspace(pa, 2, 90, d.k_cache, 8))
    st = pa.pa_get_status()
    assert st & pa.PA_STATUS_BAD_BLOCK_ID
    # context length above max_context_len: clamped and flagged
    pa.pa_decode(out, d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, 64, case.scale, 64,
                 torch.empty(pa.pa_decode_workspace_bytes(2, 64, 64, pa.shape_of(d.k_cache, 8)), dtype=torch.uint8,
                             device="cuda"))
    assert pa.pa_get_status() & pa.PA_STATUS_BAD_CONTEXT
    assert pa.pa_get_status() == 0


def test_graph_capture_replays_step(pa):
    case = W.make_case("graph", 13, context_lens=[100, 2000, 517], q_lens=[1, 1, 1], num_heads=32, num_kv_heads=8,
                       head_dim=128, dtype="bf16")
    d = DevCase(case)
    kc0, vc0 = d.k_cache.clone(), d.v_cache.clone()
    shape = pa.shape_of(d.k_cache, 32)
    ws = torch.empty(pa.pa_decode_workspace_bytes(3, 2000, 0, shape), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(d.q)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        pa.pa_reshape_and_cache(d.k_new, d.v_new, d.k_cache, d.v_cache, d.slot_mapping)
        pa.pa_decode(out, d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, 2000, case.scale, 0, ws)
    torch.cuda.synchronize()
    eager = out.clone()
    d.k_cache.copy_(kc0)
    d.v_cache.copy_(vc0)
    out.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        pa.pa_reshape_and_cache(d.k_new, d.v_new, d.k_cache, d.v_cache, d.slot_mapping)
        pa.pa_decode(out, d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, 2000, case.scale, 0, ws)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
    assert pa.pa_get_status() == 0


@pytest.mark.parametrize("name", ["decode_batch", "long_context"])
def test_slice_counts_agree(pa, name):
    # the automatic slicing and forced finer and coarser ones: every output element within the
    # tolerance of the oracle (checked elsewhere) and of each other
    case = W.CONFIGS[name]()
    d = DevCase(case)
    pa.pa_reshape_and_cache(d.k_new, d.v_new, d.k_cache, d.v_cache, d.slot_mapping)
    mx = int(case.context_lens.max())
    shape = pa.shape_of(d.k_cache, case.num_heads)
    outs = []
    for part in (0, 64, 4096):
        ws = torch.empty(max(pa.pa_decode_workspace_bytes(case.num_seqs, mx, part, shape), 16), dtype=torch.uint8,
                         device="cuda")
        o = torch.full_like(d.q, float("nan"))
        pa.pa_decode(o, d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, mx, case.scale, part, ws)
        outs.append(o.float())
    assert pa.pa_get_status() == 0
    for o in outs[1:]:
        assert torch.isfinite(o).all()
        assert (o - outs[0]).abs().max().item() <= TOL["bf16"]


def test_workspace_needs_no_initialisation(pa):
    # Every partial and record a call reads it writes first, so a workspace
    # holding random bytes, or the leftovers of a call of another geometry,
    # gives the same result as a fresh one.
    big = W.make_case("ws_big", 31, context_lens=[4000, 2500, 900, 3333, 1500, 64], q_lens=[1] * 6, num_heads=32,
                      num_kv_heads=8, head_dim=128, dtype="bf16")
    small = W.make_case("ws_small", 32, context_lens=[1200, 700, 2049], q_lens=[1] * 3, num_heads=32,
                        num_kv_heads=8, head_dim=128, dtype="bf16")
    shape_b = pa.shape_of(to_dev(big.k_cache), 32)
    n = max(pa.pa_decode_workspace_bytes(6, 4000, 128, shape_b), pa.pa_decode_workspace_bytes(3, 2049, 128, shape_b))
    g = torch.Generator(device="cuda").manual_seed(5)
    ws = torch.randint(0, 256, (n,), dtype=torch.uint8, device="cuda", generator=g)
    for case in (big, small, big):  # the second and third calls start on the earlier calls' leftovers
        d = DevCase(case)
        pa.pa_reshape_and_cache(d.k_new, d.v_new, d.k_cache, d.v_cache, d.slot_mapping)
        out = torch.full_like(d.q, float("nan"))
        mx = int(case.context_lens.max())
        pa.pa_decode(out, d.q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, mx, case.scale, 128, ws)
        assert pa.pa_get_status() == 0
        kc_ref, vc_ref = oracle_written(case)
        ref = oracle.decode(case.q, kc_ref, vc_ref, case.block_tables, case.context_lens, case.scale)
        assert max_err(to_host(out), ref) <= TOL["bf16"], case.name


def test_graph_replays_with_new_queries(pa):
    # a captured pa_decode (both kernels) replayed on new queries
    case = W.make_case("replay", 33, context_lens=[3000, 1000, 4096, 17], q_lens=[1] * 4, num_heads=32,
                       num_kv_heads=8, head_dim=128, dtype="bf16")
    d = DevCase(case)
    pa.pa_reshape_and_cache(d.k_new, d.v_new, d.k_cache, d.v_cache, d.slot_mapping)
    shape = pa.shape_of(d.k_cache, 32)
    ws = torch.zeros(pa.pa_decode_workspace_bytes(4, 4096, 256, shape), dtype=torch.uint8, device="cuda")
    q = d.q.clone()
    out = torch.empty_like(q)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        pa.pa_decode(out, q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, 4096, case.scale, 256, ws)
    s.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr, stream=s):
        pa.pa_decode(out, q, d.k_cache, d.v_cache, d.block_tables, d.context_lens, 4096, case.scale, 256, ws)
    kc_ref, vc_ref = oracle_written(case)
    rng = np.random.default_rng(34)
    for _ in range(3):
        q_np = W.f32_to_bf16_bits(rng.uniform(-1, 1, case.q.shape).astype(np.float32))
        q.copy_(to_dev(q_np))
        gr.replay()
        torch.cuda.synchronize()
        ref = oracle.decode(q_np, kc_ref, vc_ref, case.block_tables, case.context_lens, case.scale)
        assert max_err(to_host(out), ref) <= TOL["bf16"]
    assert pa.pa_get_status() == 0
