"""One serving decode step from host buffers: the end-to-end public API.

A DecodeStep owns the device-resident KV pool, the decode workspace and the
device copies of one step's inputs. A step does, in order:
  1. host->device copies of q, the new tokens' K/V, slot_mapping,
     block_tables and context_lens,
  2. pa_reshape_and_cache (the new tokens go to their slots first),
  3. pa_decode over every sequence,
  4. a device->host copy of out.
The KV pool stays on the device between steps, because it is the cache.

Inputs reach the step in one of two ways:
  * staged (the fast path): inputs() returns pinned host views of all six
    inputs, packed in one buffer. The caller writes each step's inputs there,
    and a step moves them with a single host->device copy.
  * bound: bind() takes the caller's own pinned tensors, and a step copies
    each of them (six copies).
With use_graph=True the whole step is captured once as a CUDA graph and
replayed, so each step is one launch. That is how a serving loop records a
step ("vLLM and PagedAttention", ai.zenoagi.com, §6: CUDA graphs).
"""
from __future__ import annotations

import torch

from . import pa

_ALIGN = 256  # byte alignment of each input inside the staging buffers


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
        # (name, shape, dtype) of the step's inputs, in staging order
        self._spec = [("q", (num_seqs, num_heads, d), dt), ("k_new", (num_seqs, hk, d), dt),
                      ("v_new", (num_seqs, hk, d), dt), ("slot_mapping", (num_seqs,), torch.int64),
                      ("block_tables", (num_seqs, max_blocks_per_seq), torch.int32),
                      ("context_lens", (num_seqs,), torch.int32)]
        self._offsets, off = [], 0
        for _, shape, dtype in self._spec:
            self._offsets.append(off)
            n = torch.Size(shape).numel() * torch.empty((), dtype=dtype).element_size()
            off = (off + n + _ALIGN - 1) // _ALIGN * _ALIGN
        self._stage_bytes = off
        self._stage_d = torch.empty(off, dtype=torch.uint8, device=dev)
        views = self._views(self._stage_d)
        self.q, self.k_new, self.v_new, self.slot_mapping, self.block_tables, self.context_lens = views
        self.out = torch.empty_like(self.q)
        nbytes = pa.pa_decode_workspace_bytes(num_seqs, max_context_len, partition_tokens,
                                              pa.shape_of(k_cache, num_heads, k_scale, v_scale))
        self.workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev) if nbytes else None
        self.stream = torch.cuda.Stream(device=dev)
        self.use_graph = use_graph
        self.graph = None
        self._host = None        # bound mode: the caller's six pinned tensors
        self._stage_h = None     # staged mode: one pinned buffer
        self._out_h = None

    def _views(self, buf: torch.Tensor):
        out = []
        for (_, shape, dtype), off in zip(self._spec, self._offsets):
            n = torch.Size(shape).numel() * torch.empty((), dtype=dtype).element_size()
            out.append(buf[off:off + n].view(dtype).view(shape))
        return out

    def inputs(self, out: torch.Tensor = None) -> dict:
        """Staged mode: pinned host views of the six inputs in one buffer (write them before each run()).

        `out` is the pinned host tensor run() writes the attention output to
        (allocated here when not given). Returns the views by name, and "out".
        """
        if self._stage_h is None:
            self._stage_h = torch.empty(self._stage_bytes, dtype=torch.uint8).pin_memory()
        if out is None:
            out = torch.empty(tuple(self.out.shape), dtype=self.out.dtype).pin_memory()
        elif out.is_cuda or not out.is_pinned():
            raise ValueError("out must be a pinned CPU tensor")
        self._out_h = out
        self._host = None
        self.graph = None
        views = dict(zip([s[0] for s in self._spec], self._views(self._stage_h)))
        views["out"] = out
        return views

    def h2d_bytes(self) -> int:
        if self._host is None and self._stage_h is not None:
            return self._stage_bytes
        return sum(t.numel() * t.element_size() for t in
                   (self.q, self.k_new, self.v_new, self.slot_mapping, self.block_tables, self.context_lens))

    def d2h_bytes(self) -> int:
        return self.out.numel() * self.out.element_size()

    def _enqueue(self):
        if self._host is not None:
            q, k_new, v_new, slots, tables, lens, _ = self._host
            for dst, src in zip((self.q, self.k_new, self.v_new, self.slot_mapping, self.block_tables,
                                 self.context_lens), (q, k_new, v_new, slots, tables, lens)):
                dst.copy_(src, non_blocking=True)
        else:
            self._stage_d.copy_(self._stage_h, non_blocking=True)
        pa.pa_reshape_and_cache(self.k_new, self.v_new, self.k_cache, self.v_cache, self.slot_mapping,
                                k_scale=self.k_scale, v_scale=self.v_scale)
        pa.pa_decode(self.out, self.q, self.k_cache, self.v_cache, self.block_tables, self.context_lens,
                     self.max_context_len, self.scale, self.partition_tokens, self.workspace,
                     k_scale=self.k_scale, v_scale=self.v_scale)
        self._result().copy_(self.out, non_blocking=True)

    def _result(self) -> torch.Tensor:
        return self._host[-1] if self._host is not None else self._out_h

    def bind(self, q, k_new, v_new, slot_mapping, block_tables, context_lens, out):
        """Bound mode: fix the pinned host tensors that later run() calls read and write."""
        for t in (q, k_new, v_new, slot_mapping, block_tables, context_lens, out):
            if t.is_cuda or not t.is_pinned():
                raise ValueError("host buffers must be pinned CPU tensors")
        self._host = (q, k_new, v_new, slot_mapping, block_tables, context_lens, out)
        self.graph = None

    def launch(self):
        """Enqueue one step on self.stream without waiting for it."""
        if self._host is None and (self._stage_h is None or self._out_h is None):
            raise RuntimeError("call inputs() or bind() first")
        with torch.cuda.stream(self.stream):
            if not self.use_graph:
                self._enqueue()
                return
            if self.graph is None:
                self._enqueue()  # warm-up outside capture
                self.stream.synchronize()
                self.graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(self.graph, stream=self.stream):
                    self._enqueue()
            self.graph.replay()

    def run(self):
        """One step: host inputs -> device -> write + decode -> host output; returns the host output."""
        self.launch()
        self.stream.synchronize()
        return self._result()
