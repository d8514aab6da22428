"""Helpers for the GPU parity tests: upload a PagedCase, run the library, compare with the oracle."""
from __future__ import annotations

import functools

import numpy as np
import torch

import oracle
from paged_kv_cache_366_b200 import workloads as W

TOL = {"bf16": 5e-3, "f32": 1e-5}


def to_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def to_host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def widen(a: np.ndarray) -> np.ndarray:
    if a.dtype == np.uint16:
        return W.bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


class DevCase:
    """Device copies of one case's inputs."""

    def __init__(self, case: W.PagedCase, device="cuda"):
        self.case = case
        self.k_cache = to_dev(case.k_cache, device)
        self.v_cache = to_dev(case.v_cache, device)
        self.k_new = to_dev(case.k_new, device)
        self.v_new = to_dev(case.v_new, device)
        self.q = to_dev(case.q, device)
        self.slot_mapping = to_dev(case.slot_mapping, device)
        self.block_tables = to_dev(case.block_tables, device)
        self.context_lens = to_dev(case.context_lens, device)
        self.cu_q_lens = to_dev(case.cu_q_lens, device)


def decode_rows(case: W.PagedCase, seqs) -> np.ndarray:
    """Query row (the last token) of each listed sequence."""
    return np.asarray([int(case.cu_q_lens[b + 1]) - 1 for b in seqs], dtype=np.int64)


def oracle_written(case: W.PagedCase):
    return oracle.reshape_and_cache(case.k_new, case.v_new, case.k_cache, case.v_cache, case.slot_mapping)


def max_err(gpu_out: np.ndarray, ref: np.ndarray) -> float:
    g = widen(gpu_out)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    if not np.all(np.isfinite(g)):
        return float("inf")
    return float(np.abs(g - ref).max()) if g.size else 0.0


@functools.lru_cache(maxsize=1)
def mixed_step_reference():
    """The mixed step (a 2048-token chunk at offset 6144 and 192 decode tokens) with the oracle's
    written caches and its attention for every one of the 2240 query rows, computed once per
    test session."""
    case = W.mixed_step()
    kc, vc = oracle_written(case)
    ref = oracle.prefill(case.q, kc, vc, case.block_tables, case.cu_q_lens, case.context_lens, case.scale)
    return case, ref


def decode_workspace(pa, num_seqs, max_context_len, k_cache, num_heads, partition_tokens=0, k_scale=0.0,
                     v_scale=0.0):
    """A workspace of the size pa_decode asks for (uninitialised: pa_decode needs none)."""
    n = pa.pa_decode_workspace_bytes(num_seqs, max_context_len, partition_tokens,
                                     pa.shape_of(k_cache, num_heads, k_scale, v_scale))
    return torch.empty(max(n, 16), dtype=torch.uint8, device=k_cache.device)
