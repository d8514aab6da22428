"""CPU-only checks: the C ABI's exports and host-side argument handling, and bench.py's host logic."""
import ctypes
import json
import os
import re
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_ \*]*?\b(pa_[a-z0-9_]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_function():
    from paged_kv_cache_366_b200 import pa
    names = declared_functions()
    assert "pa_decode" in names and "pa_reshape_and_cache" in names and "pa_prefill_chunk" in names
    lib = ctypes.CDLL(pa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(pa.EXPORTED) == set(names)


def test_abi_version_and_messages():
    from paged_kv_cache_366_b200 import pa
    assert pa.pa_abi_version() == 7
    assert pa.pa_strerror(0) == "ok"
    assert "workspace" in pa.pa_strerror(-4)
    assert pa.pa_strerror(-99) == "unknown error"


def shape(**kw):
    from paged_kv_cache_366_b200 import pa
    d = dict(num_heads=32, num_kv_heads=8, head_dim=128, block_size=16, num_blocks=1000, dtype=1)
    d.update(kw)
    return pa.PaShape(**d)


def r16(n):
    return (n + 15) // 16 * 16


def ws_bytes(B, ctas, H=32, Hk=8, D=128, warps=12):
    """Workspace of a decode over `ctas` CTAs (one slice per warp, 12 warps for bf16 32/8 heads of 128):
    partial O, m and l per slot (slice + unit), then an int32 (first slice, slices) record per unit."""
    units = B * Hk
    slots = warps * ctas + units - 1
    g = H // Hk
    return slots * g * D * 4 + 2 * r16(slots * g * 4) + r16(units * 8)


def test_workspace_sizes():
    from paged_kv_cache_366_b200 import pa
    s = shape()
    assert pa.pa_decode_workspace_bytes(0, 2048, 0, s) == 0
    # one CTA (the list has 8 blocks at most)
    assert pa.pa_decode_workspace_bytes(1, 16, 0, s) == ws_bytes(1, 1)
    # forced: slices of about 512 tokens of a 2048-token context: 64 * 8 * 128 * 16 / 512 = 2048
    # slices, 171 CTAs of 12
    assert pa.pa_decode_workspace_bytes(64, 2048, 512, s) == ws_bytes(64, 171)
    with pytest.raises(pa.PaError):
        pa.pa_decode_workspace_bytes(4, 100, 100, s)  # not a multiple of 64


def test_automatic_slices():
    # no GPU here, so the policy assumes 148 SMs holding one decode CTA of 12 warps each: 1776 slices
    from paged_kv_cache_366_b200 import pa
    s = shape()
    assert pa.pa_decode_workspace_bytes(64, 2048, 0, s) == ws_bytes(64, 148)
    assert pa.pa_decode_workspace_bytes(8, 32768, 0, s) == ws_bytes(8, 148)
    assert pa.pa_decode_workspace_bytes(256, 2016, 0, s) == ws_bytes(256, 148)
    # one sequence of 4096 tokens: 8 * 256 blocks at most, one slice per 4 blocks: 512 slices, 43 CTAs
    assert pa.pa_decode_workspace_bytes(1, 4096, 0, s) == ws_bytes(1, 43)


@pytest.mark.parametrize("kw,code", [
    (dict(block_size=32), -2), (dict(head_dim=96), -2), (dict(num_heads=24, num_kv_heads=8), -2),
    (dict(num_heads=30, num_kv_heads=8), -1), (dict(dtype=7), -2), (dict(num_blocks=0), -1),
])
def test_shape_validation(kw, code):
    from paged_kv_cache_366_b200 import pa
    s = shape(**kw)
    assert pa.lib.pa_decode_workspace_bytes(4, 100, 0, ctypes.byref(s)) == code


@pytest.mark.parametrize("kw,code", [
    (dict(kv_fp8=1, k_scale=0.1, v_scale=0.1), 0), (dict(kv_fp8=1, k_scale=0.0, v_scale=0.1), -1),
    (dict(kv_fp8=1, k_scale=0.1, v_scale=float("inf")), -1), (dict(kv_fp8=1, dtype=0, k_scale=1.0, v_scale=1.0), -2),
    (dict(kv_fp8=2), -1),
])
def test_fp8_cache_shape_validation(kw, code):
    from paged_kv_cache_366_b200 import pa
    s = shape(**kw)
    rc = pa.lib.pa_decode_workspace_bytes(4, 100, 0, ctypes.byref(s))
    assert (rc >= 0) if code == 0 else rc == code


def test_null_pointers_are_rejected_before_any_launch():
    from paged_kv_cache_366_b200 import pa
    s = shape()
    assert pa.lib.pa_decode(None, None, None, None, None, 4, None, 2, 64, 1.0, 0, None, 0, ctypes.byref(s),
                            None) == -1
    rc = pa.lib.pa_reshape_and_cache(None, None, None, None, None, 3, ctypes.byref(s), None)
    assert rc == -1
    assert pa.lib.pa_reshape_and_cache(None, None, None, None, None, 0, ctypes.byref(s), None) == 0
    rc = pa.lib.pa_prefill_chunk(None, None, None, None, None, 4, None, None, 1, 8, 8, 1.0, ctypes.byref(s), None)
    assert rc == -1
    s32 = shape(dtype=0)
    rc = pa.lib.pa_prefill_chunk(None, None, None, None, None, 4, None, None, 1, 8, 8, 1.0, ctypes.byref(s32), None)
    assert rc == -2  # prefill is bf16 only


def test_empty_inputs_are_no_ops():
    """Empty batches return success before any check that needs a pointer, and launch nothing (the
    calls below run on a machine without a GPU)."""
    from paged_kv_cache_366_b200 import pa
    s = shape()
    by = ctypes.byref(s)
    assert pa.lib.pa_reshape_and_cache(None, None, None, None, None, 0, by, None) == 0
    for fn in (pa.lib.pa_decode, pa.lib.pa_decode_partials, pa.lib.pa_decode_merge):
        assert fn(None, None, None, None, None, 4, None, 0, 64, 1.0, 0, None, 0, by, None) == 0
    assert pa.lib.pa_decode_noalloc(None, None, None, None, None, 4, None, 0, 64, 1.0, 0, by, None) == 0
    # no sequences, or sequences with no query tokens
    assert pa.lib.pa_prefill_chunk(None, None, None, None, None, 4, None, None, 0, 8, 8, 1.0, by, None) == 0
    assert pa.lib.pa_prefill_chunk(None, None, None, None, None, 4, None, None, 2, 0, 0, 1.0, by, None) == 0
    assert pa.lib.pa_copy_blocks(None, None, None, 0, by, None) == 0
    assert pa.lib.pa_swap_blocks(None, None, None, 0, 4, 4, 16 * 8 * 128 * 2, None) == 0
    # negative sizes are errors, not no-ops
    assert pa.lib.pa_reshape_and_cache(None, None, None, None, None, -1, by, None) == -1
    assert pa.lib.pa_decode(None, None, None, None, None, 4, None, -1, 64, 1.0, 0, None, 0, by, None) == -1
    assert pa.lib.pa_copy_blocks(None, None, None, -1, by, None) == -1


def test_misaligned_pointer_is_rejected():
    from paged_kv_cache_366_b200 import pa
    s = shape()
    p = ctypes.c_void_p(0x1000 + 8)
    ok = ctypes.c_void_p(0x2000)
    rc = pa.lib.pa_reshape_and_cache(p, ok, ok, ok, ok, 3, ctypes.byref(s), None)
    assert rc == -3


def test_bench_step_bytes_and_split():
    import bench
    from paged_kv_cache_366_b200 import workloads as W
    case = W.make_case("x", 1, context_lens=[20, 300, 17], q_lens=[5, 1, 1], num_heads=8, num_kv_heads=2,
                       head_dim=64, dtype="bf16")
    dec, pre = bench.split_seqs(case)
    assert list(dec) == [1, 2] and list(pre) == [0]
    b = bench.step_bytes(case, dec, pre)
    assert b["kv_decode"] == (300 + 17) * 2 * 64 * 2 * 2
    assert b["write"] == 7 * 2 * 64 * 2 * 4 + 7 * 8
    assert b["total"] == b["write"] + b["decode"] + b["prefill"]
    # causal chunk of 5 at offset 15: keys 16..20 per query
    assert bench.prefill_flops(case, pre) == sum(range(16, 21)) * 8 * 64 * 4


def test_bench_reads_profiled_traffic_only_for_matching_sources(tmp_path, monkeypatch):
    import bench
    (tmp_path / "profiles").mkdir()
    sha = bench.decode_source_sha()
    (tmp_path / "profiles" / "decode_kernel_w.md").write_text(
        "# summary\n\n- traffic_bytes_per_launch: 123456\n- source_sha256: %s\n" % sha)
    (tmp_path / "profiles" / "decode_kernel_stale.md").write_text(
        "- traffic_bytes_per_launch: 7\n- source_sha256: %s\n" % ("0" * 64))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "decode_source_sha", lambda sources=None: sha)
    assert bench.profiled_traffic("w") == 123456.0
    assert bench.profiled_traffic("stale") is None
    assert bench.profiled_traffic("missing") is None


def test_bench_reference_arm_runs_on_cpu():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "tiny", "--steps", "3", "--warmup", "3"], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "GB/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def _agg_worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    b, t = bench.aggregate(100.0 * (rank + 1), 1.0 + rank)
    q.put((rank, b, t))
    dist.destroy_process_group()


def test_bench_aggregate_two_ranks_gloo():
    import multiprocessing as mp
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ps = [ctx.Process(target=_agg_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    # bytes summed over replicas, time is the slowest replica's
    assert res == [(0, 300.0, 2.0), (1, 300.0, 2.0)]
