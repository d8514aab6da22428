"""Python binding of libpa.so: the C ABI in include/pa.h, same names.

Argument marshalling only. Each call checks that its tensors are CUDA,
contiguous and of the expected dtype, passes their pointers and the current
torch stream to the C entry point, and raises PaError on a nonzero return.
Every step of the computation runs in the library's kernels. There is no
fallback: if libpa.so is missing, importing this module raises ImportError.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

PA_DTYPE_F32, PA_DTYPE_BF16 = 0, 1
BLOCK_SIZE = 16

PA_STATUS_BAD_BLOCK_ID = 0x1
PA_STATUS_BAD_SLOT = 0x2
PA_STATUS_BAD_CONTEXT = 0x4
PA_STATUS_WAIT_TIMEOUT = 0x8
PA_STATUS_BAD_QUERY = 0x10
PA_ABI_VERSION = 7


class PaShape(ctypes.Structure):
    _fields_ = [
        ("num_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("num_blocks", ctypes.c_int64),
        ("dtype", ctypes.c_int32),
        ("kv_fp8", ctypes.c_int32),
        ("k_scale", ctypes.c_float),
        ("v_scale", ctypes.c_float),
    ]


EXPORTED = [
    "pa_reshape_and_cache", "pa_decode_workspace_bytes", "pa_decode", "pa_decode_partials", "pa_decode_merge",
    "pa_prefill_chunk",
    "pa_get_status", "pa_strerror", "pa_last_cuda_error", "pa_abi_version", "pa_decode_noalloc",
    "pa_copy_blocks", "pa_swap_blocks",
]

PA_ERR_SCRATCH_LIMIT = -7
PA_NOALLOC_SCRATCH_BYTES = 16 << 20


def _load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError("libpa.so not built at %s: run paged_kv_cache_366_b200/build.py" % path)
    lib = ctypes.CDLL(path)
    P, I32, I64, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    SP = ctypes.POINTER(PaShape)
    lib.pa_reshape_and_cache.argtypes = [P, P, P, P, P, I64, SP, P]
    lib.pa_reshape_and_cache.restype = ctypes.c_int
    lib.pa_decode_workspace_bytes.argtypes = [I32, I32, I32, SP]
    lib.pa_decode_workspace_bytes.restype = I64
    for name in ("pa_decode", "pa_decode_partials", "pa_decode_merge"):
        getattr(lib, name).argtypes = [P, P, P, P, P, I32, P, I32, I32, F, I32, P, I64, SP, P]
        getattr(lib, name).restype = ctypes.c_int
    lib.pa_prefill_chunk.argtypes = [P, P, P, P, P, I32, P, P, I32, I32, I32, F, SP, P]
    lib.pa_prefill_chunk.restype = ctypes.c_int
    lib.pa_decode_noalloc.argtypes = [P, P, P, P, P, I32, P, I32, I32, F, I32, SP, P]
    lib.pa_decode_noalloc.restype = ctypes.c_int
    lib.pa_copy_blocks.argtypes = [P, P, P, I64, SP, P]
    lib.pa_copy_blocks.restype = ctypes.c_int
    lib.pa_swap_blocks.argtypes = [P, P, P, I64, I64, I64, I64, P]
    lib.pa_swap_blocks.restype = ctypes.c_int
    lib.pa_get_status.argtypes = [ctypes.POINTER(ctypes.c_uint32), P]
    lib.pa_get_status.restype = ctypes.c_int
    lib.pa_strerror.argtypes = [ctypes.c_int]
    lib.pa_strerror.restype = ctypes.c_char_p
    lib.pa_last_cuda_error.argtypes = []
    lib.pa_last_cuda_error.restype = ctypes.c_int
    lib.pa_abi_version.argtypes = []
    lib.pa_abi_version.restype = ctypes.c_int
    return lib


lib = _load()
if lib.pa_abi_version() != PA_ABI_VERSION:
    raise ImportError("libpa.so has ABI version %d, the binding expects %d: rebuild it"
                      % (lib.pa_abi_version(), PA_ABI_VERSION))


class PaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        msg = "%s: %s (%d)" % (fn, lib.pa_strerror(code).decode(), code)
        if code == -5:
            msg += ", cudaError %d" % lib.pa_last_cuda_error()
        super().__init__(msg)


def _check(fn: str, rc: int) -> None:
    if rc != 0:
        raise PaError(fn, rc)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return PA_DTYPE_BF16
    if dt == torch.float32:
        return PA_DTYPE_F32
    raise ValueError("dtype must be bfloat16 or float32, got %s" % dt)


def shape_of(k_cache: torch.Tensor, num_heads: int, k_scale: float = 0.0, v_scale: float = 0.0) -> PaShape:
    """pa_shape of a pool [NB, 16, Hk, D] read by `num_heads` query heads.

    A uint8 pool holds FP8 E4M3 codes (values code * k_scale / code * v_scale)
    next to bf16 q/out and new tokens.
    """
    if k_cache.dim() != 4:
        raise ValueError("k_cache must be [num_blocks, block_size, num_kv_heads, head_dim]")
    nb, bs, hk, d = k_cache.shape
    fp8 = k_cache.dtype == torch.uint8
    return PaShape(num_heads=int(num_heads), num_kv_heads=int(hk), head_dim=int(d), block_size=int(bs),
                   num_blocks=int(nb), dtype=PA_DTYPE_BF16 if fp8 else _dtype_code(k_cache.dtype),
                   kv_fp8=1 if fp8 else 0, k_scale=float(k_scale), v_scale=float(v_scale))


def _same_dtype_kv(q_like, caches):
    """q/out/new tokens share one dtype; caches share it or are uint8 FP8 codes with bf16 elsewhere."""
    _same_dtype(*q_like)
    _same_dtype(*caches)
    if caches[0].dtype == torch.uint8:
        if q_like[0].dtype != torch.bfloat16:
            raise ValueError("an FP8 cache goes with bf16 q, out and new tokens")
    elif caches[0].dtype != q_like[0].dtype:
        raise ValueError("q/out/k/v and the caches must share one dtype")


def _same_dtype(*ts):
    dts = {t.dtype for t in ts}
    if len(dts) != 1:
        raise ValueError("q/k/v/caches/out must share one dtype, got %s" % sorted(map(str, dts)))


def _int(t: torch.Tensor, dt: torch.dtype, name: str):
    if t.dtype != dt:
        raise ValueError("%s must be %s" % (name, dt))


def pa_reshape_and_cache(k, v, k_cache, v_cache, slot_mapping, stream=None, k_scale: float = 0.0,
                         v_scale: float = 0.0) -> None:
    """Write each new token's K/V row into its slot of the pool (bit-exact copy, or FP8 quantization)."""
    _same_dtype_kv((k, v), (k_cache, v_cache))
    _int(slot_mapping, torch.int64, "slot_mapping")
    shape = shape_of(k_cache, k_cache.shape[2], k_scale, v_scale)
    if k.shape[1:] != k_cache.shape[2:] or v.shape != k.shape or slot_mapping.shape[0] != k.shape[0]:
        raise ValueError("k, v must be [T, Hk, D] matching the cache; slot_mapping [T]")
    _check("pa_reshape_and_cache",
           lib.pa_reshape_and_cache(_ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping),
                                    k.shape[0], ctypes.byref(shape), _stream(stream)))


def pa_decode_workspace_bytes(num_seqs: int, max_context_len: int, partition_tokens: int, shape: PaShape) -> int:
    n = lib.pa_decode_workspace_bytes(int(num_seqs), int(max_context_len), int(partition_tokens),
                                      ctypes.byref(shape))
    if n < 0:
        raise PaError("pa_decode_workspace_bytes", int(n))
    return int(n)


def _decode(fn: str, out, q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale,
            partition_tokens, workspace, stream, k_scale, v_scale) -> None:
    _same_dtype_kv((out, q), (k_cache, v_cache))
    _int(block_tables, torch.int32, "block_tables")
    _int(context_lens, torch.int32, "context_lens")
    B, H, D = q.shape
    if out.shape != q.shape or block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("q, out [B, H, D]; block_tables [B, MB]; context_lens [B]")
    shape = shape_of(k_cache, H, k_scale, v_scale)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(fn,
           getattr(lib, fn)(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                            block_tables.shape[1], _ptr(context_lens), B, int(max_context_len), float(scale),
                            int(partition_tokens), _ptr(workspace), ws_bytes, ctypes.byref(shape),
                            _stream(stream)))


def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len: int, scale: float,
              partition_tokens: int = 0, workspace: Optional[torch.Tensor] = None, stream=None,
              k_scale: float = 0.0, v_scale: float = 0.0) -> None:
    """Decode attention of one query token per sequence over its paged context."""
    _decode("pa_decode", out, q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale,
            partition_tokens, workspace, stream, k_scale, v_scale)


def pa_decode_partials(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len: int, scale: float,
                       partition_tokens: int = 0, workspace: Optional[torch.Tensor] = None, stream=None,
                       k_scale: float = 0.0, v_scale: float = 0.0) -> None:
    """The first of pa_decode's two launches: the partition pass (arguments as pa_decode)."""
    _decode("pa_decode_partials", out, q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale,
            partition_tokens, workspace, stream, k_scale, v_scale)


def pa_decode_merge(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len: int, scale: float,
                    partition_tokens: int = 0, workspace: Optional[torch.Tensor] = None, stream=None,
                    k_scale: float = 0.0, v_scale: float = 0.0) -> None:
    """The second of pa_decode's two launches: the merge of cut units (arguments as pa_decode)."""
    _decode("pa_decode_merge", out, q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale,
            partition_tokens, workspace, stream, k_scale, v_scale)


def pa_decode_noalloc(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len: int, scale: float,
                      partition_tokens: int = 0, stream=None, k_scale: float = 0.0, v_scale: float = 0.0) -> None:
    """pa_decode without a workspace argument, for callers that cannot allocate device memory.

    The split-context partials go to a PA_NOALLOC_SCRATCH_BYTES array built
    into the library (held on every device that loads it). Requests that need
    more raise PaError with PA_ERR_SCRATCH_LIMIT. Calls that may overlap on
    one GPU share that array and must not run concurrently. Make the first
    call on each device outside stream capture. A uint8 (FP8 E4M3) pool takes
    k_scale and v_scale as in pa_decode.
    """
    _same_dtype_kv((out, q), (k_cache, v_cache))
    _int(block_tables, torch.int32, "block_tables")
    _int(context_lens, torch.int32, "context_lens")
    B, H, D = q.shape
    if out.shape != q.shape or block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("q, out [B, H, D]; block_tables [B, MB]; context_lens [B]")
    shape = shape_of(k_cache, H, k_scale, v_scale)
    _check("pa_decode_noalloc",
           lib.pa_decode_noalloc(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                 block_tables.shape[1], _ptr(context_lens), B, int(max_context_len), float(scale),
                                 int(partition_tokens), ctypes.byref(shape), _stream(stream)))


def pa_prefill_chunk(out, q, k_cache, v_cache, block_tables, cu_q_lens, context_lens, max_q_len: int,
                     scale: float, stream=None, k_scale: float = 0.0, v_scale: float = 0.0) -> None:
    """Causal attention of query chunks at their context offsets (bf16 q/out, D=128; bf16 caches, or uint8
    FP8 E4M3 caches with their k_scale / v_scale)."""
    _same_dtype_kv((out, q), (k_cache, v_cache))
    _int(block_tables, torch.int32, "block_tables")
    _int(cu_q_lens, torch.int32, "cu_q_lens")
    _int(context_lens, torch.int32, "context_lens")
    T, H, D = q.shape
    B = context_lens.shape[0]
    if out.shape != q.shape or block_tables.shape[0] != B or cu_q_lens.shape[0] != B + 1:
        raise ValueError("q, out [T, H, D]; block_tables [B, MB]; cu_q_lens [B+1]; context_lens [B]")
    shape = shape_of(k_cache, H, k_scale, v_scale)
    _check("pa_prefill_chunk",
           lib.pa_prefill_chunk(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                block_tables.shape[1], _ptr(cu_q_lens), _ptr(context_lens), B, int(max_q_len), T,
                                float(scale), ctypes.byref(shape), _stream(stream)))


def pa_copy_blocks(k_cache, v_cache, block_pairs, stream=None) -> None:
    """Copy whole blocks inside the pool: block_pairs int64 [n, 2] of (src, dst), on the device."""
    _same_dtype(k_cache, v_cache)
    _int(block_pairs, torch.int64, "block_pairs")
    shape = shape_of(k_cache, k_cache.shape[2], 1.0, 1.0)
    _check("pa_copy_blocks", lib.pa_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(block_pairs),
                                                block_pairs.numel() // 2, ctypes.byref(shape), _stream(stream)))


def _any_ptr(t: torch.Tensor):
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    if not t.is_cuda and not t.is_pinned():
        raise ValueError("host tensors must be pinned")
    return ctypes.c_void_p(t.data_ptr())


def pa_swap_blocks(dst, src, block_pairs, stream=None) -> None:
    """Copy blocks of one pool between device and pinned host memory: block_pairs int64 [n, 2] of (src, dst)."""
    if dst.dtype != src.dtype or dst.shape[1:] != src.shape[1:]:
        raise ValueError("dst and src pools must have the same dtype and block shape")
    _int(block_pairs, torch.int64, "block_pairs")
    bb = src[0].numel() * src.element_size()
    _check("pa_swap_blocks", lib.pa_swap_blocks(_any_ptr(dst), _any_ptr(src), _any_ptr(block_pairs),
                                                block_pairs.numel() // 2, src.shape[0], dst.shape[0], bb,
                                                _stream(stream)))


def pa_get_status(stream=None) -> int:
    """Synchronize the stream, return and clear the device status word (PA_STATUS_* flags)."""
    v = ctypes.c_uint32(0)
    _check("pa_get_status", lib.pa_get_status(ctypes.byref(v), _stream(stream)))
    return int(v.value)


def pa_strerror(code: int) -> str:
    return lib.pa_strerror(int(code)).decode()


def pa_abi_version() -> int:
    return int(lib.pa_abi_version())
