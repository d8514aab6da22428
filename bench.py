#!/usr/bin/env python3
"""Benchmark of the paged-KV attention hot path on B200.

One step is the whole path for one batch: the KV write of this step's new
tokens (pa_reshape_and_cache), then paged decode over every decode sequence
(pa_decode: one kernel, the split-context pass with the merge of split
contexts fused in). The mixed workload also runs the causal prefill chunk
(pa_prefill_chunk). Inputs are synthetic, seeded and resident in HBM before
the timed region. Each step is captured once as CUDA graphs and replayed
between CUDA events on the launching stream. Before every step, outside the
events, a 256 MiB memset and then a 256 MiB read flush L2 (the read makes the
memset's dirty lines drain to HBM before the step starts).

Output: one JSON line on rank 0. `value` is the step's algorithmic bytes
over the step time, in GB/s and summed over ranks (N > 1 runs independent
replicas, with no data exchange). `roofline` rates the decode call (its
algorithmic bytes over its event time) against the measured HBM copy
bandwidth, and against the nominal 8000 GB/s. `e2e` times the public
DecodeStep API from pinned host buffers, with the copies inside.
`cpu_baseline` is the fp64 oracle on the host cores. On the decode batch the
line also carries, under `also`, the long-context decode, the prefill chunk,
decode and the chunk over an FP8 pool, prefix sharing, a batch of verify
chunks, the mixed step as two launches and as one, and the block copy and
swap, each with its own roofline and clocks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from paged_kv_cache_366_b200 import workloads as W  # noqa: E402

METRIC = "paged decode attention KV GB/s and % of B200 HBM peak; decode tokens/s"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
FLUSH_BYTES = 256 << 20
DECODE_SOURCES = ["decode.cuh", "pa_common.cuh", "tmap.cuh"]
PREFILL_SOURCES = ["prefill_sm100.cuh", "pa_common.cuh", "tmap.cuh"]
WORKLOADS = ["decode_batch", "long_context", "prefix_sharing", "mixed_step", "prefill_chunk", "tiny",
             "copy_blocks", "swap_blocks", "decode_batch_fp8", "prefill_chunk_fp8", "varlen_step", "spec_verify"]
FP8_K_SCALE, FP8_V_SCALE = 0.02, 1.0 / 48.0
BLOCK_WORKLOADS = ("copy_blocks", "swap_blocks")
BLOCK_PAIRS = 2048


# ---------------------------------------------------------------------------
# Workload bookkeeping (host side)

def split_seqs(case):
    """Decode sequences (one new token) and prefill sequences (a chunk), each a contiguous range."""
    ql = case.q_lens
    dec = np.nonzero(ql == 1)[0]
    pre = np.nonzero(ql > 1)[0]
    for r in (dec, pre):
        if len(r):
            assert np.array_equal(r, np.arange(r[0], r[-1] + 1)), "decode/prefill sequences must be contiguous"
    return dec, pre


def step_bytes(case, dec, pre, kv_elem=None):
    """Algorithmic bytes of one step, by part (kv_elem: bytes per cache element, default the case's)."""
    E, H, Hk, D = case.elem_bytes, case.num_heads, case.num_kv_heads, case.head_dim
    KE = E if kv_elem is None else kv_elem
    ctx = case.context_lens.astype(np.int64)
    T = case.num_tokens
    write = T * Hk * D * (E + KE) * 2 + T * 8
    kv_dec = int(ctx[dec].sum()) * Hk * D * KE * 2
    tables_dec = int(((ctx[dec] + 15) // 16).sum()) * 4 + 4 * len(dec)
    decode = kv_dec + len(dec) * H * D * E * 2 + tables_dec
    prefill = 0
    if len(pre):
        qt = int(case.q_lens[pre].sum())
        prefill = int(ctx[pre].sum()) * Hk * D * E * 2 + qt * H * D * E * 2 + int(((ctx[pre] + 15) // 16).sum()) * 4
    return {"write": write, "decode": decode, "kv_decode": kv_dec, "prefill": prefill,
            "total": write + decode + prefill}


def prefill_flops(case, pre):
    H, D = case.num_heads, case.head_dim
    f = 0
    for b in pre:
        c, q = int(case.context_lens[b]), int(case.q_lens[b])
        o = c - q
        f += sum((o + j + 1) for j in range(q)) * H * D * 4
    return f


def describe(case, dec, pre):
    ctx = case.context_lens
    d = {"workload": case.name, "num_seqs": int(case.num_seqs), "num_heads": case.num_heads,
         "num_kv_heads": case.num_kv_heads, "head_dim": case.head_dim, "block_size": case.block_size,
         "kv_dtype": case.dtype, "pool_blocks": int(case.num_blocks), "seed": case.seed,
         "decode_seqs": int(len(dec)), "new_tokens": int(case.num_tokens),
         "context_len_mean": float(ctx[dec].mean()) if len(dec) else 0.0,
         "context_len_range": [int(ctx.min()), int(ctx.max())]}
    if len(pre):
        d["prefill_query_tokens"] = int(case.q_lens[pre].sum())
    return d


FALLBACK_BF16_TFLOPS = 1590.0


def load_peak(key="hbm_gbs"):
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)[key]), "measured"
    except Exception:
        return (FALLBACK_HBM_GBS if key == "hbm_gbs" else FALLBACK_BF16_TFLOPS), "fallback"


def decode_source_sha(sources=None):
    h = hashlib.sha256()
    for n in sources or DECODE_SOURCES:
        with open(os.path.join(ROOT, "paged_kv_cache_366_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profiled_traffic(workload, kernel="decode_kernel", sources=None):
    """dram read+write bytes per launch from the committed ncu summary, if it matches the source."""
    path = os.path.join(ROOT, "profiles", "%s_%s.md" % (kernel, workload))
    try:
        kv = {}
        with open(path) as f:
            for line in f:
                item = line.strip().lstrip("-* `")  # markdown list items: "- key: value"
                if ":" in item and item.startswith(("traffic_bytes_per_launch", "source_sha256")):
                    k, v = item.split(":", 1)
                    kv[k.strip().strip("`")] = v.strip().strip("` ")
        if kv.get("source_sha256") == decode_source_sha(sources):
            return float(kv["traffic_bytes_per_launch"])
    except Exception:
        pass
    return None


# ---------------------------------------------------------------------------
# Clock sampling during the timed regions

REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


class ClockSampler:
    """nvidia-smi samples (every 50 ms) of SM clocks and throttle reasons, summarised per time window."""

    def __init__(self, gpu: str):
        self.samples = []
        self.proc = None
        q = ("timestamp,clocks.sm,clocks.max.sm,power.draw," +
             ",".join("clocks_event_reasons." + r for r in REASONS))
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", gpu, "--query-gpu=" + q,
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 4 + len(REASONS):
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                self.samples.append((ts, float(parts[1]), float(parts[2]),
                                     [r for r, v in zip(REASONS, parts[4:]) if v.lower() == "active"]))
            except ValueError:
                continue

    def wait_ready(self, timeout=5.0):
        t0 = time.time()
        while self.proc and not self.samples and time.time() - t0 < timeout:
            time.sleep(0.05)

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.proc = None

    def window(self, t0, t1):
        """Median SM clock, max clock and throttle reasons of the samples taken in [t0, t1]."""
        if not self.samples:
            return None
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside:  # region shorter than the sampling period: nearest samples
            inside = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:2]
        reasons = sorted({r for s in inside for r in s[3]})
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": max(s[2] for s in inside),
                "reasons": reasons, "samples": len(inside)}


def gpu_id_for(local_rank: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# ---------------------------------------------------------------------------
# Multi-rank plumbing (replicas: only timing and byte counts cross ranks)

def aggregate(local_bytes: float, local_seconds: float):
    """(sum of bytes over ranks, max of seconds over ranks); identity without a process group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return local_bytes, local_seconds
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    b = torch.tensor([local_bytes], dtype=torch.float64, device=dev)
    t = torch.tensor([local_seconds], dtype=torch.float64, device=dev)
    dist.all_reduce(b, op=dist.ReduceOp.SUM)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(b.item()), float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ---------------------------------------------------------------------------
# CPU oracle: the cpu_baseline leg and the reference arm

def oracle_sample_seqs(case):
    """Sequences the oracle samples: the decode sequences, or every sequence of a chunk-only workload."""
    dec, _ = split_seqs(case)
    return dec if len(dec) else np.arange(case.num_seqs)


def oracle_step(case, seqs, num_threads, caches=None):
    """The oracle on the listed sequences: cache write of all their new tokens, then decode of each
    sequence's last token (the query that attends to its whole context). With `caches` (writable copies
    of the pool) the write lands in place, as the GPU's does; otherwise the oracle returns new copies."""
    import oracle
    written = np.concatenate([np.arange(int(case.cu_q_lens[b]), int(case.cu_q_lens[b + 1])) for b in seqs])
    rows = np.asarray([int(case.cu_q_lens[b + 1]) - 1 for b in seqs], dtype=np.int64)
    kc, vc = caches if caches is not None else (case.k_cache, case.v_cache)
    kc, vc = oracle.reshape_and_cache(case.k_new[written], case.v_new[written], kc, vc,
                                      case.slot_mapping[written], in_place=caches is not None)
    oracle.decode(case.q[rows], kc, vc, case.block_tables[seqs], case.context_lens[seqs], case.scale,
                  num_threads=num_threads)


def step_bytes_for(case, seqs):
    """Algorithmic bytes of oracle_step on these sequences: the write, then one decode query each."""
    E, H, Hk, D = case.elem_bytes, case.num_heads, case.num_kv_heads, case.head_dim
    ctx = case.context_lens[seqs].astype(np.int64)
    n = len(seqs)
    t = int(case.q_lens[seqs].astype(np.int64).sum())  # tokens written
    return (t * Hk * D * E * 4 + t * 8 + int(ctx.sum()) * Hk * D * E * 2 + n * H * D * E * 2 +
            int(((ctx + 15) // 16).sum()) * 4 + 4 * n)


def host_cores():
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


def time_oracle(case, budget_s, min_reps=1, threads=None, n_seqs=None):
    """Oracle throughput on a bounded sample of the workload's decode sequences; returns a dict."""
    dec = oracle_sample_seqs(case)
    cores = threads or host_cores()
    caches = (np.array(case.k_cache, copy=True), np.array(case.v_cache, copy=True))
    if n_seqs:
        n = min(len(dec), n_seqs)
    else:
        t0 = time.perf_counter()
        oracle_step(case, dec[:1], cores, caches)
        t_one = max(time.perf_counter() - t0, 1e-4)
        n = int(max(1, min(len(dec), budget_s / t_one)))
    seqs = dec[:n]
    reps, spent = 0, 0.0
    while reps < min_reps or spent < budget_s * 0.5:
        t0 = time.perf_counter()
        oracle_step(case, seqs, cores, caches)
        spent += time.perf_counter() - t0
        reps += 1
        if spent > budget_s:
            break
    nbytes = step_bytes_for(case, seqs) * reps
    return {"value": nbytes / spent / 1e9, "unit": UNIT, "cores": int(cores), "kind": "oracle",
            "sample": "fp64 C oracle (OpenMP, %d threads): cache write (in place) + decode of the first %d of %d "
                      "sequences of %s, %d repetition(s), %.2f s" % (cores, n, len(dec), case.name, reps, spent),
            "seconds": spent, "n_seqs": n}


def run_reference(args):
    """The oracle, as it stands, on the host cores: each step writes the step's new tokens in place
    and decodes every sampled sequence. All sequences are taken when (warmup + steps) of them fit in
    about four minutes (the decode batch does at the default step count on 16 host cores), else the
    first n that do."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    case = make_workload(args.workload)
    dec = oracle_sample_seqs(case)
    cores = host_cores()
    caches = (np.array(case.k_cache, copy=True), np.array(case.v_cache, copy=True))
    budget = max(0.005, 240.0 / (args.steps + args.warmup))  # about four minutes in all
    t0 = time.perf_counter()
    oracle_step(case, dec, cores, caches)
    t_all = max(time.perf_counter() - t0, 1e-4)
    n = len(dec) if t_all <= budget else int(max(1, len(dec) * budget / t_all))
    seqs = dec[:n]
    for _ in range(args.warmup):
        oracle_step(case, seqs, cores, caches)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(case, seqs, cores, caches)
    dt = time.perf_counter() - t0
    nbytes = step_bytes_for(case, seqs) * args.steps
    value = nbytes / dt / 1e9
    config = describe(case, *split_seqs(case))
    config["sampled_seqs"] = int(n)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": int(cores), "kind": "oracle",
                             "sample": "fp64 C oracle: each step = cache write (in place) of the step's new tokens "
                                       "+ decode of %s%d of %d sequences of %s (for chunks: all their tokens "
                                       "written, the last token's query attended)" % (
                                           "all " if n == len(dec) else "the first ", n, len(dec), case.name)},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm

# Workloads whose whole attention is one pa_prefill_chunk launch over every
# sequence (decode tokens as chunks of 1, verify chunks, prefill chunks).
ONE_LAUNCH = ("varlen_step", "spec_verify")
NOMINAL_HBM_GBS = 8000.0  # the nominal HBM peak the targets are quoted against
# Companions of the decode-batch line: the other target config (long context), the tensor-core
# chunk, the FP8 pool (decode and the chunk), prefix sharing, a one-launch batch of verify chunks,
# and the mixed step as two launches and as one, each timed in the same run with its own roofline
# and clocks.
ALSO = ("long_context", "prefill_chunk", "decode_batch_fp8", "prefill_chunk_fp8", "prefix_sharing", "spec_verify",
        "mixed_step", "varlen_step")


def make_workload(name):
    if name.endswith("_fp8"):  # the same sequences over a pool of E4M3 codes
        name = name[:-len("_fp8")]
    if name == "varlen_step":  # the mixed step's sequences, attended in one launch
        return W.mixed_step()
    if name not in W.CONFIGS:
        raise SystemExit("unknown workload %s (one of %s)" % (name, ", ".join(WORKLOADS)))
    return W.CONFIGS[name]()


def unique_kv_bytes(case, dec):
    """K/V bytes of the distinct physical rows the decode sequences read (shared blocks counted once)."""
    Hk, D, E = case.num_kv_heads, case.head_dim, case.elem_bytes
    rows = {}
    for b in dec:
        c = int(case.context_lens[b])
        for i in range((c + 15) // 16):
            pb = int(case.block_tables[b, i])
            rows[pb] = max(rows.get(pb, 0), min(16, c - 16 * i))
    return sum(rows.values()) * Hk * D * E * 2


class Flush:
    """Evict L2 between timed steps: write a buffer larger than L2, then read another, so the write's
    dirty lines reach HBM before the timed events rather than during them."""

    def __init__(self):
        import torch
        self.w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        self.r = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")

    def __call__(self):
        import torch
        self.w.zero_()
        torch.sum(self.r)


def measure_gpu(name, steps, warmup, flush, sampler, want_e2e):
    """Set up one workload on the device, capture its step and parts as CUDA graphs, and time them.

    Returns a dict with the case, the step's algorithmic bytes by part, the summed step time (seconds over
    `steps` steps), the per-part times per step, clocks during the step loop and the e2e figures."""
    import torch
    from paged_kv_cache_366_b200 import pa
    from paged_kv_cache_366_b200.step import DecodeStep

    def dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(a)).cuda()

    case = make_workload(name)
    dec, pre = split_seqs(case)
    fp8 = name.endswith("_fp8")
    ks, vs = (FP8_K_SCALE, FP8_V_SCALE) if fp8 else (0.0, 0.0)
    nbytes = step_bytes(case, dec, pre, 1 if fp8 else None)

    k_cache, v_cache = dev(case.k_cache), dev(case.v_cache)
    if fp8:  # quantize the whole pool with the library's own FP8 write
        NB, bs, Hk, D = case.k_cache.shape
        kc8 = torch.empty(tuple(k_cache.shape), dtype=torch.uint8, device="cuda")
        vc8 = torch.empty_like(kc8)
        every_slot = torch.arange(NB * bs, dtype=torch.int64, device="cuda")
        pa.pa_reshape_and_cache(k_cache.view(NB * bs, Hk, D), v_cache.view(NB * bs, Hk, D), kc8, vc8, every_slot,
                                k_scale=ks, v_scale=vs)
        torch.cuda.synchronize()
        del k_cache, v_cache, every_slot
        k_cache, v_cache = kc8, vc8
    k_new, v_new, q = dev(case.k_new), dev(case.v_new), dev(case.q)
    slots = dev(case.slot_mapping)
    tables, lens, cu = dev(case.block_tables), dev(case.context_lens), dev(case.cu_q_lens)
    shape = pa.shape_of(k_cache, case.num_heads, ks, vs)

    d0, d1 = (int(dec[0]), int(dec[-1]) + 1) if len(dec) else (0, 0)
    dec_rows = torch.from_numpy(np.asarray([int(case.cu_q_lens[b + 1]) - 1 for b in dec], np.int64)).cuda()
    q_dec = q.index_select(0, dec_rows).contiguous() if len(dec) else None
    out_dec = torch.empty_like(q_dec) if len(dec) else None
    max_ctx = int(case.context_lens[dec].max()) if len(dec) else 0
    ws_n = pa.pa_decode_workspace_bytes(len(dec), max_ctx, 0, shape) if len(dec) else 0
    ws = torch.empty(max(ws_n, 16), dtype=torch.uint8, device="cuda") if ws_n else None

    if len(pre):
        p0, p1 = int(pre[0]), int(pre[-1]) + 1
        r0, r1 = int(case.cu_q_lens[p0]), int(case.cu_q_lens[p1])
        q_pre = q[r0:r1].contiguous()
        out_pre = torch.empty_like(q_pre)
        cu_pre = (cu[p0:p1 + 1] - int(case.cu_q_lens[p0])).contiguous()
        max_q = int(case.q_lens[pre].max())

    stream = torch.cuda.Stream()

    def do_write():
        pa.pa_reshape_and_cache(k_new, v_new, k_cache, v_cache, slots, k_scale=ks, v_scale=vs)

    def do_decode():  # the partition pass, then the merge of cut units (a programmatic dependent)
        pa.pa_decode(out_dec, q_dec, k_cache, v_cache, tables[d0:d1], lens[d0:d1], max_ctx, case.scale, 0, ws,
                     k_scale=ks, v_scale=vs)

    def do_partials():  # the partition pass alone: decode_kernel, the dominant kernel
        pa.pa_decode_partials(out_dec, q_dec, k_cache, v_cache, tables[d0:d1], lens[d0:d1], max_ctx, case.scale, 0,
                              ws, k_scale=ks, v_scale=vs)

    def do_merge():  # the merge alone, on the partials the pass before it left in the workspace
        pa.pa_decode_merge(out_dec, q_dec, k_cache, v_cache, tables[d0:d1], lens[d0:d1], max_ctx, case.scale, 0,
                           ws, k_scale=ks, v_scale=vs)


    def do_prefill():
        pa.pa_prefill_chunk(out_pre, q_pre, k_cache, v_cache, tables[p0:p1], cu_pre, lens[p0:p1], max_q,
                            case.scale, k_scale=ks, v_scale=vs)

    one = name in ONE_LAUNCH
    out_all = torch.empty_like(q)
    max_q_all = int(case.q_lens.max())

    def do_all():  # every sequence's chunk, decode tokens included, in one launch
        pa.pa_prefill_chunk(out_all, q, k_cache, v_cache, tables, cu, lens, max_q_all, case.scale, k_scale=ks,
                            v_scale=vs)

    parts = [("write", do_write)]
    extra = []
    if one:
        parts.append(("attention", do_all))
    else:
        if len(pre):
            parts.append(("prefill", do_prefill))
        if len(dec):
            parts.append(("decode", do_decode))
            extra += [("decode_kernel", do_partials), ("merge_kernel", do_merge)]
    launches_per_step = len(parts) + (1 if len(dec) and not one else 0)  # pa_decode launches two kernels

    # one graph for the whole step (the headline), one per part (breakdown, roofline)
    graphs = []
    with torch.cuda.stream(stream):
        for _, fn in parts + extra:  # eager once, then capture
            fn()
        stream.synchronize()
        for _, fn in parts + extra:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                fn()
            graphs.append(g)
        g_step = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_step, stream=stream):
            for _, fn in parts:
                fn()
    torch.cuda.synchronize()
    status = pa.pa_get_status(stream)
    if status:
        raise SystemExit("device status 0x%x after the first step of %s" % (status, name))

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            flush()
            g_step.replay()
            flush()
            for g in graphs:
                g.replay()
    torch.cuda.synchronize()

    # timed region: `steps` steps, each one graph replay between events, L2 flushed before each
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier()
    torch.cuda.synchronize()
    wall0 = time.time()
    with torch.cuda.stream(stream):
        for i in range(steps):
            flush()
            step_ev[i][0].record(stream)
            g_step.replay()
            step_ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    wall1 = time.time()
    status = pa.pa_get_status(stream)
    if status:
        raise SystemExit("device status 0x%x after the timed steps of %s" % (status, name))
    total = sum(a.elapsed_time(b) for a, b in step_ev) * 1e-3

    # per-part times (each part its own graph, events between), for the breakdown and rooflines
    n_parts_steps = min(steps, 500)
    names = [n for n, _ in parts + extra]
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * len(graphs))] for _ in range(n_parts_steps)]
    with torch.cuda.stream(stream):
        for i in range(n_parts_steps):
            for j, g in enumerate(graphs):
                flush()
                events[i][2 * j].record(stream)
                g.replay()
                events[i][2 * j + 1].record(stream)
    torch.cuda.synchronize()
    per_part = {n: sum(ev[2 * j].elapsed_time(ev[2 * j + 1]) for ev in events) * 1e-3 / n_parts_steps
                for j, n in enumerate(names)}  # seconds per step
    clocks = sampler.window(wall0, wall1) if sampler else None

    # end to end through the public API, host buffers, copies inside (decode workloads)
    e2e = None
    if want_e2e and len(dec) and not len(pre):
        step = DecodeStep(k_cache, v_cache, case.num_heads, len(dec), case.max_blocks_per_seq, max_ctx,
                          case.scale, k_scale=ks, v_scale=vs)
        rows = np.asarray([int(case.cu_q_lens[b + 1]) - 1 for b in dec], np.int64)
        views = step.inputs()  # staged inputs: the step's six inputs in one pinned buffer

        def fill(dst, a):
            a = np.ascontiguousarray(a)
            src = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
            (dst.view(torch.int16) if a.dtype == np.uint16 else dst).copy_(src)
        fill(views["q"], case.q[rows])
        fill(views["k_new"], case.k_new[rows])
        fill(views["v_new"], case.v_new[rows])
        fill(views["slot_mapping"], case.slot_mapping[rows])
        fill(views["block_tables"], case.block_tables[d0:d1])
        fill(views["context_lens"], case.context_lens[d0:d1])
        n_e2e = max(10, min(steps, 500))
        for _ in range(max(3, warmup)):
            step.run()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_e2e)]
        barrier()
        for i in range(n_e2e):
            with torch.cuda.stream(step.stream):
                flush()
                ev[i][0].record(step.stream)
            step.launch()
            with torch.cuda.stream(step.stream):
                ev[i][1].record(step.stream)
            step.stream.synchronize()
        barrier()
        t_e2e = sum(a.elapsed_time(b) for a, b in ev) * 1e-3
        b_e2e, t_e2e = aggregate(float(nbytes["total"]) * n_e2e, t_e2e)
        e2e = {"value": b_e2e / t_e2e / 1e9, "unit": UNIT, "h2d_bytes_per_step": step.h2d_bytes(),
               "d2h_bytes_per_step": step.d2h_bytes(), "steps": n_e2e, "ms_per_step": t_e2e / n_e2e * 1e3,
               "api": "paged_kv_cache_366_b200.step.DecodeStep, staged inputs (one copy in, one out; CUDA graph)"}
    del graphs, g_step
    return {"case": case, "dec": dec, "pre": pre, "nbytes": nbytes, "total": total, "per_part": per_part,
            "clocks": clocks, "e2e": e2e, "one": one, "fp8": fp8, "ks": ks, "vs": vs,
            "launches_per_step": launches_per_step, "wall": (wall0, wall1)}


def decode_roofline(m, peak, peak_kind, name):
    """Roofline of the dominant decode kernel, decode_kernel (pa_decode_partials, timed alone), with the whole
    pa_decode call (the kernel and the merge of cut units) beside it."""
    t_dec = m["per_part"]["decode_kernel"]
    t_call = m["per_part"]["decode"]
    nb = m["nbytes"]["decode"]
    achieved = nb / t_dec / 1e9
    r = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
         "frac_of_nominal": achieved / NOMINAL_HBM_GBS, "nominal_peak": NOMINAL_HBM_GBS,
         "traffic": profiled_traffic(name), "kernel": "decode_kernel (pa_decode_partials: the partition pass, "
                                                      "one CTA of 12 warps per SM, one slice per warp)",
         "algorithmic_bytes_per_launch": nb, "us_per_launch": t_dec * 1e6,
         "merge_us_per_launch": m["per_part"]["merge_kernel"] * 1e6,
         "pa_decode_call": {"us": t_call * 1e6, "achieved": nb / t_call / 1e9, "frac": nb / t_call / 1e9 / peak,
                            "frac_of_nominal": nb / t_call / 1e9 / NOMINAL_HBM_GBS},
         "peak_kind": peak_kind + " (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else peak_kind}
    return r


def prefill_roofline(m, name):
    case, pre = m["case"], m["pre"]
    f = prefill_flops(case, pre)
    t_pre = m["per_part"]["prefill"]
    tpeak, tkind = load_peak("bf16_tflops")
    tf = f / t_pre / 1e12
    return {"bound": "tensor", "achieved": tf, "peak": tpeak, "unit": "TFLOP/s", "frac": tf / tpeak,
            "traffic": profiled_traffic(name, "prefill_kernel", PREFILL_SOURCES), "kernel": "prefill_kernel (tcgen05)",
            "flops_per_launch": f, "us_per_launch": t_pre * 1e6,
            "peak_kind": tkind + " bf16 burst (MEASURED_PEAKS.json bf16_tflops)"}


def one_launch_roofline(m, peak, peak_kind):
    """One launch does the decode tokens (HBM-bound) and the chunks (tensor-bound when long). Its floor
    is the chunks' FLOPs at the bf16 peak plus the decode tokens' bytes at the copy bandwidth; a launch
    of verify chunks alone is HBM-bound (a few rows per KV head)."""
    case, dec, pre, nbytes = m["case"], m["dec"], m["pre"], m["nbytes"]
    t_one = m["per_part"]["attention"]
    tpeak, tkind = load_peak("bf16_tflops")
    f = prefill_flops(case, pre)
    attn_bytes = nbytes["decode"] + nbytes["prefill"]
    long_chunks = [b for b in pre if int(case.q_lens[b]) > 64]
    f_long = prefill_flops(case, long_chunks)
    short_bytes = attn_bytes - (step_bytes(case, dec, np.asarray(long_chunks, np.int64))["prefill"]
                                if long_chunks else 0)
    t_floor = f_long / (tpeak * 1e12) + short_bytes / (peak * 1e9)
    roof = {"bound": "hbm" if not long_chunks else "hbm+tensor",
            "achieved": attn_bytes / t_one / 1e9 if not long_chunks else t_floor / t_one,
            "peak": peak if not long_chunks else 1.0,
            "unit": "GB/s" if not long_chunks else "fraction of the summed floor",
            "frac": t_floor / t_one, "traffic": None,
            "kernel": "prefill_kernel (tcgen05), one launch over every sequence",
            "algorithmic_bytes_per_launch": attn_bytes, "flops_per_launch": f,
            "floor_us": t_floor * 1e6, "us_per_launch": t_one * 1e6,
            "peak_kind": "%s (MEASURED_PEAKS.json hbm_gbs%s)" % (
                peak_kind, "" if not long_chunks else " and bf16_tflops, " + tkind)}
    if not long_chunks:
        roof["frac_of_nominal"] = attn_bytes / t_one / 1e9 / NOMINAL_HBM_GBS
    return roof


def unique_bytes_entry(m, peak):
    """Prefix sharing: the decode's K/V bytes counting each shared physical row once."""
    case, dec, nbytes = m["case"], m["dec"], m["nbytes"]
    ub = unique_kv_bytes(case, dec) + (nbytes["decode"] - nbytes["kv_decode"])
    t_dec = m["per_part"]["decode"]
    return {"decode_bytes": ub, "gbs": ub / t_dec / 1e9, "frac": ub / t_dec / 1e9 / peak,
            "frac_of_nominal": ub / t_dec / 1e9 / NOMINAL_HBM_GBS,
            "note": "K/V bytes of the distinct physical rows read (the shared prefix once), "
                    "plus q, out and tables, over the pa_decode time"}


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        raise SystemExit("--gpus %d but WORLD_SIZE %d" % (args.gpus, world))
    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))

    sampler = ClockSampler(gpu_id_for(local_rank)) if rank == 0 else None
    if sampler:
        sampler.wait_ready()
    flush = Flush()
    m = measure_gpu(args.workload, args.steps, args.warmup, flush, sampler, want_e2e=True)
    case, dec, pre, nbytes = m["case"], m["dec"], m["pre"], m["nbytes"]
    sum_bytes, t_max = aggregate(float(nbytes["total"]) * args.steps, m["total"])
    value = sum_bytes / t_max / 1e9
    ms_per_step = t_max / args.steps * 1e3

    # companions of the headline in the same run (ALSO), each with its own roofline and clocks
    also = {}
    if not args.no_also and args.workload == "decode_batch":
        peak, peak_kind = load_peak()
        for extra in ALSO:
            torch.cuda.empty_cache()
            steps_x = max(5, min(args.steps, 50))
            mx = measure_gpu(extra, steps_x, args.warmup, flush, sampler, want_e2e=False)
            b_x, t_x = aggregate(float(mx["nbytes"]["total"]) * steps_x, mx["total"])
            ent = {"steps": steps_x, "ms_per_step": t_x / steps_x * 1e3, "value": b_x / t_x / 1e9, "unit": UNIT,
                   "pct_of_hbm_peak": b_x / t_x / 1e9 / peak,
                   "pct_of_nominal_peak": b_x / t_x / 1e9 / NOMINAL_HBM_GBS,
                   "clocks": mx["clocks"], "config": describe(mx["case"], mx["dec"], mx["pre"])}
            if mx["fp8"]:
                ent["config"].update({"workload": extra, "kv_dtype": "fp8_e4m3", "k_scale": mx["ks"],
                                      "v_scale": mx["vs"]})
            if mx["one"]:
                ent["roofline"] = one_launch_roofline(mx, peak, peak_kind)
            elif len(mx["dec"]):
                ent["roofline"] = decode_roofline(mx, peak, peak_kind, extra)
            elif len(mx["pre"]):
                ent["roofline"] = prefill_roofline(mx, extra)
            if extra.startswith("prefix_sharing"):
                ent["unique_bytes"] = unique_bytes_entry(mx, peak)
            also[extra] = ent
            del mx
        for extra in BLOCK_WORKLOADS:
            torch.cuda.empty_cache()
            bl = measure_blocks(extra, max(5, min(args.steps, 50)), args.warmup, sampler)
            also[extra] = {k: bl[k] for k in ("steps", "ms_per_step", "value", "unit", "clocks", "config", "roofline")}

    if world > 1:
        dist.destroy_process_group()
    if sampler:
        sampler.stop()
    if rank != 0:
        return 0

    peak, peak_kind = load_peak()
    per_part = m["per_part"]
    roof = None
    if not m["one"] and len(dec):
        roof = decode_roofline(m, peak, peak_kind, args.workload)
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        cpu = time_oracle(case, args.cpu_seconds)
        # the same oracle and sample on one thread (one repetition at least)
        single = time_oracle(case, max(1.0, args.cpu_seconds / 4), threads=1, n_seqs=cpu["n_seqs"])
        cpu["single_thread"] = {"value": single["value"], "unit": single["unit"], "cores": 1,
                                "sample": single["sample"]}
        cpu.pop("seconds", None)
        cpu.pop("n_seqs", None)
    parts_ms = {k: v * 1e3 for k, v in per_part.items()}
    config = describe(case, dec, pre)
    if m["fp8"]:
        config.update({"workload": args.workload, "kv_dtype": "fp8_e4m3", "k_scale": m["ks"],
                       "v_scale": m["vs"]})
    config.update({"l2": "flushed before every step and every timed part, outside the events: 256 MiB memset, "
                         "then a 256 MiB read so the memset's write-back is not charged to the step",
                   "timing": "one CUDA graph replay per step between CUDA events on the launching stream; "
                             "per-part times from a second loop of per-part graphs",
                   "parallelism": "replicas" if args.gpus > 1 else "single GPU",
                   "global_batch": int(case.num_seqs) * args.gpus})
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": case.dtype, "data": "synthetic (seeded; see paged_kv_cache_366_b200/"
                                                                 "workloads.py)",
            "config": config, "pct_of_hbm_peak": value / peak, "pct_of_nominal_peak": value / NOMINAL_HBM_GBS,
            "decode_tokens_per_s": len(dec) * args.gpus / (t_max / args.steps),
            "kv_gbs": nbytes["kv_decode"] * args.gpus / (t_max / args.steps) / 1e9,
            "ms_per_part": parts_ms, "step_bytes": nbytes, "roofline": roof, "cpu_baseline": cpu, "e2e": m["e2e"],
            "clocks": m["clocks"], "gpu_launches": m["launches_per_step"] * args.steps,
            "wall_s_timed_region": m["wall"][1] - m["wall"][0]}
    if args.workload.startswith("prefix_sharing"):
        line["unique_bytes"] = unique_bytes_entry(m, peak)
    if m["one"]:
        line["roofline"] = one_launch_roofline(m, peak, peak_kind)
    if not m["one"] and len(pre):
        pr = prefill_roofline(m, args.workload)
        line["prefill"] = {"flops": pr["flops_per_launch"], "us_per_launch": pr["us_per_launch"],
                           "tflops": pr["achieved"], "roofline": pr}
        if not len(dec):
            line["roofline"] = pr
    if also:
        line["also"] = also
    print(json.dumps(line), flush=True)
    return 0


def run_blocks(args):
    """Whole-block copies on the decode-batch pool (see measure_blocks): one JSON line."""
    if int(os.environ.get("WORLD_SIZE", "1")) > 1 and int(os.environ.get("RANK", "0")) != 0:
        return 0  # replicas of a copy measure nothing the single run does not
    print(json.dumps(measure_blocks(args.workload, args.steps, args.warmup)), flush=True)
    return 0


def measure_blocks(workload, steps, warmup, sampler=None):
    """Whole-block copies on the decode-batch pool; returns the bench line.

    copy_blocks: copy-on-write of 2048 (used -> free) blocks, K and V, inside HBM.
    swap_blocks: 2048 blocks of K and V out to pinned host memory and back in,
    one pa_swap_blocks launch per pool and direction.
    """
    import torch
    from paged_kv_cache_366_b200 import pa

    case = W.decode_batch()
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    k_cache, v_cache = dev(case.k_cache), dev(case.v_cache)
    rng = np.random.default_rng(17)
    used = np.unique(case.block_tables[case.block_tables >= 0])
    free = np.setdiff1d(np.arange(case.num_blocks), used)
    n = min(BLOCK_PAIRS, len(free))
    block_bytes = k_cache[0].numel() * 2
    stream = torch.cuda.Stream()
    flush_w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    flush_r = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    if workload == "copy_blocks":
        pairs = torch.from_numpy(np.stack([rng.choice(used, n), rng.choice(free, n, replace=False)], 1)
                                 .astype(np.int64)).cuda()
        fns = [lambda: pa.pa_copy_blocks(k_cache, v_cache, pairs)]
        nbytes = n * 2 * 2 * block_bytes
        launches = 2
        peak, kind = load_peak()
        bound, peak_note = "hbm", kind + " (MEASURED_PEAKS.json hbm_gbs)"
    else:
        src_ids = rng.choice(used, n, replace=False)
        host_k = torch.empty((n,) + tuple(k_cache.shape[1:]), dtype=torch.bfloat16).pin_memory()
        host_v = torch.empty_like(host_k).pin_memory()
        out_pairs = torch.from_numpy(np.stack([src_ids, np.arange(n)], 1).astype(np.int64)).cuda()
        in_pairs = torch.from_numpy(np.stack([np.arange(n), rng.choice(free, n, replace=False)], 1)
                                    .astype(np.int64)).cuda()
        fns = [lambda: (pa.pa_swap_blocks(host_k, k_cache, out_pairs), pa.pa_swap_blocks(host_v, v_cache, out_pairs),
                        pa.pa_swap_blocks(k_cache, host_k, in_pairs), pa.pa_swap_blocks(v_cache, host_v, in_pairs))]
        nbytes = n * 2 * 2 * block_bytes  # out and back in, K and V, over the host link
        launches = 4
        # link reference, measured here: contiguous pinned copies of the same bytes, out and in
        dbuf = torch.empty(n * block_bytes, dtype=torch.uint8, device="cuda")
        hbuf = torch.empty(n * block_bytes, dtype=torch.uint8).pin_memory()
        ts = []
        with torch.cuda.stream(stream):
            for i in range(6):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for _ in range(2):
                    hbuf.copy_(dbuf, non_blocking=True)
                    dbuf.copy_(hbuf, non_blocking=True)
                e1.record(stream)
                stream.synchronize()
                if i >= 2:
                    ts.append(e0.elapsed_time(e1) * 1e-3)
        peak = 4 * n * block_bytes / statistics.median(ts) / 1e9
        bound, peak_note = "link", "measured in this run: contiguous pinned cudaMemcpyAsync, same bytes, out and in"
    with torch.cuda.stream(stream):
        for f in fns:
            f()
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for f in fns:
                f()
        for _ in range(warmup):
            flush_w.zero_()
            torch.sum(flush_r)
            g.replay()
    torch.cuda.synchronize()
    if pa.pa_get_status(stream):
        raise SystemExit("device status set by the block copies")
    own_sampler = sampler is None
    if own_sampler:
        sampler = ClockSampler(gpu_id_for(int(os.environ.get("LOCAL_RANK", "0"))))
        sampler.wait_ready()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    wall0 = time.time()
    with torch.cuda.stream(stream):
        for a, b in ev:
            flush_w.zero_()
            torch.sum(flush_r)
            a.record(stream)
            g.replay()
            b.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    clocks = sampler.window(wall0, wall1)
    if own_sampler:
        sampler.stop()
    del g
    t = sum(a.elapsed_time(b) for a, b in ev) * 1e-3 / steps
    value = nbytes / t / 1e9
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": steps, "warmup": warmup,
            "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; see paged_kv_cache_366_b200/workloads.py)",
            "config": {"workload": workload, "pool": "decode_batch (seed 1)", "block_pairs": n,
                       "block_bytes_per_pool": block_bytes,
                       "l2": "flushed before every step, outside the events (memset then read)"},
            "roofline": {"bound": bound, "achieved": value, "peak": peak, "unit": "GB/s", "frac": value / peak,
                         "traffic": None, "kernel": "copy_blocks_kernel", "peak_kind": peak_note},
            "cpu_baseline": None, "e2e": None, "clocks": clocks, "gpu_launches": launches * steps}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="decode_batch", choices=WORKLOADS)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-also", action="store_true", help="skip the long-context and prefill companions")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="budget of the oracle timing")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        if args.workload in BLOCK_WORKLOADS:
            raise SystemExit("the reference arm times the attention step; block copies have no oracle timing")
        return run_reference(args)
    if args.workload in BLOCK_WORKLOADS:
        return run_blocks(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
