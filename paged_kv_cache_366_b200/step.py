"""One serving decode step from host buffers: the end-to-end public API.

A DecodeStep owns the device-resident KV pool, the decode workspace and
device staging for one step's inputs. run() takes this step's inputs in
pinned host memory and returns the attention output in pinned host memory.
In order, it does:
  1. host->device copies of q, the new tokens' K/V, slot_mapping,
     block_tables and context_lens,
  2. pa_reshape_and_cache (the new tokens go to their slots first),
  3. pa_decode over every sequence,
  4. a device->host copy of out.
The KV pool stays on the device between steps, because it is the cache.
With use_graph=True the whole sequence is captured once as a CUDA graph and
replayed, so each step is one launch. That is how a serving loop records a
step ("vLLM and PagedAttention", ai.zenoagi.com, §6: CUDA graphs).
"""
from __future__ import annotations

import torch

from . import pa


class DecodeStep:
    def __init__(self, k_cache: torch.Tensor, v_cache: torch.Tensor, num_heads: int, num_seqs: int,
                 max_blocks_per_seq: int, max_context_len: int, scale: float, partition_tokens: int = 0,
                 use_graph: bool = True, k_scale: float = 0.0, v_scale: float = 0.0):
        if not (k_cache.is_cuda and v_cache.is_cuda):
            raise ValueError("the KV pool lives on the device")
        self.k_cache, self.v_cache = k_cache, v_cache
        self.k_scale, self.v_scale = k_scale, v_scale  # for a uint8 (FP8 E4M3) pool
        dev = k_cache.device
        dt = torch.bfloat16 if k_cache.dtype == torch.uint8 else k_cache.dtype
        _, _, hk, d = k_cache.shape
        self.num_heads, self.num_seqs = num_heads, num_seqs
        self.max_context_len, self.scale, self.partition_tokens = max_context_len, scale, partition_tokens
        self.q = torch.empty((num_seqs, num_heads, d), dtype=dt, device=dev)
        self.out = torch.empty_like(self.q)
        self.k_new = torch.empty((num_seqs, hk, d), dtype=dt, device=dev)
        self.v_new = torch.empty_like(self.k_new)
        self.slot_mapping = torch.empty(num_seqs, dtype=torch.int64, device=dev)
        self.block_tables = torch.empty((num_seqs, max_blocks_per_seq), dtype=torch.int32, device=dev)
        self.context_lens = torch.empty(num_seqs, dtype=torch.int32, device=dev)
        nbytes = pa.pa_decode_workspace_bytes(num_seqs, max_context_len, partition_tokens,
                                              pa.shape_of(k_cache, num_heads, k_scale, v_scale))
        self.workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev) if nbytes else None
        self.stream = torch.cuda.Stream(device=dev)
        self.use_graph = use_graph
        self.graph = None
        self._host = None

    def h2d_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in
                   (self.q, self.k_new, self.v_new, self.slot_mapping, self.block_tables, self.context_lens))

    def d2h_bytes(self) -> int:
        return self.out.numel() * self.out.element_size()

    def _enqueue(self, host):
        q, k_new, v_new, slots, tables, lens, out = host
        self.q.copy_(q, non_blocking=True)
        self.k_new.copy_(k_new, non_blocking=True)
        self.v_new.copy_(v_new, non_blocking=True)
        self.slot_mapping.copy_(slots, non_blocking=True)
        self.block_tables.copy_(tables, non_blocking=True)
        self.context_lens.copy_(lens, non_blocking=True)
        pa.pa_reshape_and_cache(self.k_new, self.v_new, self.k_cache, self.v_cache, self.slot_mapping,
                                k_scale=self.k_scale, v_scale=self.v_scale)
        pa.pa_decode(self.out, self.q, self.k_cache, self.v_cache, self.block_tables, self.context_lens,
                     self.max_context_len, self.scale, self.partition_tokens, self.workspace,
                     k_scale=self.k_scale, v_scale=self.v_scale)
        out.copy_(self.out, non_blocking=True)

    def bind(self, q, k_new, v_new, slot_mapping, block_tables, context_lens, out):
        """Fix the pinned host buffers that later run() calls read and write (needed for graph replay)."""
        for t in (q, k_new, v_new, slot_mapping, block_tables, context_lens, out):
            if t.is_cuda or not t.is_pinned():
                raise ValueError("host buffers must be pinned CPU tensors")
        self._host = (q, k_new, v_new, slot_mapping, block_tables, context_lens, out)
        self.graph = None

    def launch(self):
        """Enqueue one step on self.stream without waiting for it."""
        if self._host is None:
            raise RuntimeError("bind() host buffers first")
        with torch.cuda.stream(self.stream):
            if not self.use_graph:
                self._enqueue(self._host)
                return
            if self.graph is None:
                self._enqueue(self._host)  # warm-up outside capture
                self.stream.synchronize()
                self.graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(self.graph, stream=self.stream):
                    self._enqueue(self._host)
            self.graph.replay()

    def run(self):
        """One step: host inputs -> device -> write + decode -> host output; returns the host output."""
        self.launch()
        self.stream.synchronize()
        return self._host[-1]
