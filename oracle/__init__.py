"""fp64 CPU oracle for paged-KV attention: a ctypes wrapper over pa_oracle.c.

TEST INFRASTRUCTURE ONLY. It is used by tests/, by the smoke check and by
bench.py's CPU-baseline and reference legs. The CUDA library never calls it,
and it never calls the CUDA library. Inputs are numpy arrays (bf16 as uint16
bit patterns) and outputs are fp64 numpy arrays. What each function computes,
and the passages it follows, is in the header comment of pa_oracle.c.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16, FP8_E4M3 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile pa_oracle.c into oracle/liboracle.so with gcc and OpenMP."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-Wextra",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P, I, L, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_long, ctypes.c_double
            lib.pa_oracle_decode.argtypes = [P, P, P, P, I, P, I, P, I, I, I, I, I, L, D, I]
            lib.pa_oracle_decode.restype = I
            lib.pa_oracle_prefill.argtypes = [P, P, P, P, I, P, I, P, P, I, I, I, I, I, L, D, P, L, I]
            lib.pa_oracle_prefill.restype = I
            lib.pa_oracle_reshape_and_cache.argtypes = [P, P, P, P, P, L, L, L]
            lib.pa_oracle_reshape_and_cache.restype = L
            lib.pa_oracle_gather.argtypes = [P, P, P, P, I, P, I, I, L, I, I, I, I, L]
            lib.pa_oracle_gather.restype = I
            lib.pa_oracle_slot_of.argtypes = [P, L, I]
            lib.pa_oracle_slot_of.restype = L
            lib.pa_oracle_blocks_for.argtypes = [L, I]
            lib.pa_oracle_blocks_for.restype = L
            lib.pa_oracle_copy_blocks.argtypes = [P, P, P, L, L, L]
            lib.pa_oracle_copy_blocks.restype = I
            lib.pa_oracle_swap_blocks.argtypes = [P, P, P, L, L, L, L]
            lib.pa_oracle_swap_blocks.restype = I
            lib.pa_oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.pa_oracle_e4m3_decode.restype = D
            lib.pa_oracle_e4m3_encode.argtypes = [ctypes.c_float]
            lib.pa_oracle_e4m3_encode.restype = ctypes.c_uint8
            lib.pa_oracle_reshape_and_cache_fp8.argtypes = [P, P, P, P, P, L, L, L, ctypes.c_float, ctypes.c_float]
            lib.pa_oracle_reshape_and_cache_fp8.restype = L
            lib.pa_oracle_decode_fp8.argtypes = [P, P, I, P, P, D, D, P, I, P, I, I, I, I, I, L, D, I]
            lib.pa_oracle_decode_fp8.restype = I
            lib.pa_oracle_prefill_fp8.argtypes = [P, P, I, P, P, D, D, P, I, P, P, I, I, I, I, I, L, D, P, L, I]
            lib.pa_oracle_prefill_fp8.restype = I
            lib.pa_oracle_set_mutation.argtypes = [I]
            lib.pa_oracle_set_mutation.restype = None
            lib.pa_oracle_get_mutation.argtypes = []
            lib.pa_oracle_get_mutation.restype = I
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.float32:
        return F32
    raise TypeError("oracle inputs are float32 or bf16 bit patterns (uint16), got %s" % a.dtype)


def _c(a, dtype=None):
    return np.ascontiguousarray(a, dtype=dtype)


class OracleError(RuntimeError):
    pass


def set_mutation(m: int) -> None:
    """Plant a known mistake in the oracle (test hook; 0 restores it)."""
    _load().pa_oracle_set_mutation(int(m))


def get_mutation() -> int:
    return int(_load().pa_oracle_get_mutation())


def blocks_for(n_tokens: int, block_size: int = 16) -> int:
    return int(_load().pa_oracle_blocks_for(int(n_tokens), int(block_size)))


def slot_of(table_row, position: int, block_size: int = 16) -> int:
    row = _c(table_row, np.int32)
    return int(_load().pa_oracle_slot_of(_ptr(row), int(position), int(block_size)))


def gather(k_cache, v_cache, block_tables, seq: int, n: int, kv_head: int, block_size: int = 16):
    """Contiguous fp64 K, V [n, D] of one sequence and KV head."""
    k_cache = _c(k_cache)
    v_cache = _c(v_cache)
    bt = _c(block_tables, np.int32)
    NB, bs, Hk, D = k_cache.shape
    assert bs == block_size
    K = np.empty((max(n, 1), D), np.float64)
    V = np.empty((max(n, 1), D), np.float64)
    rc = _load().pa_oracle_gather(_ptr(K), _ptr(V), _ptr(k_cache), _ptr(v_cache), _dtype_code(k_cache),
                                  _ptr(bt), bt.shape[1], int(seq), int(n), Hk, int(kv_head), D,
                                  block_size, NB)
    if rc:
        raise OracleError("gather failed (%d)" % rc)
    return K[:n], V[:n]


def decode(q, k_cache, v_cache, block_tables, context_lens, scale: float, num_threads: int = 0):
    """out [B, H, D] fp64 = softmax(scale q K^T) V over each sequence's gathered context."""
    q = _c(q)
    k_cache = _c(k_cache)
    v_cache = _c(v_cache)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    B, H, D = q.shape
    NB, bs, Hk, D2 = k_cache.shape
    assert D == D2 and q.dtype == k_cache.dtype == v_cache.dtype and bt.shape[0] == B == cl.shape[0]
    out = np.zeros((B, H, D), np.float64)
    rc = _load().pa_oracle_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _dtype_code(q),
                                  _ptr(bt), bt.shape[1], _ptr(cl), B, H, Hk, D, bs, NB, float(scale),
                                  int(num_threads))
    if rc:
        raise OracleError("decode failed (%d)" % rc)
    return out


def prefill(q, k_cache, v_cache, block_tables, cu_q_lens, context_lens, scale: float, rows=None,
            num_threads: int = 0):
    """Causal chunk attention. out [T or len(rows), H, D] fp64."""
    q = _c(q)
    k_cache = _c(k_cache)
    v_cache = _c(v_cache)
    bt = _c(block_tables, np.int32)
    cu = _c(cu_q_lens, np.int32)
    cl = _c(context_lens, np.int32)
    T, H, D = q.shape
    NB, bs, Hk, D2 = k_cache.shape
    B = cl.shape[0]
    assert D == D2 and cu.shape[0] == B + 1 and int(cu[-1]) == T and bt.shape[0] == B
    if rows is None:
        rows_arr, n_rows, rows_p = None, T, None
    else:
        rows_arr = _c(rows, np.int32)
        n_rows = rows_arr.shape[0]
        rows_p = _ptr(rows_arr)
    out = np.zeros((n_rows, H, D), np.float64)
    rc = _load().pa_oracle_prefill(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _dtype_code(q),
                                   _ptr(bt), bt.shape[1], _ptr(cu), _ptr(cl), B, H, Hk, D, bs, NB,
                                   float(scale), rows_p, n_rows, int(num_threads))
    if rc:
        raise OracleError("prefill failed (%d)" % rc)
    return out


def reshape_and_cache(k, v, k_cache, v_cache, slot_mapping, in_place: bool = False):
    """Return copies of (k_cache, v_cache) with each new token's row written to its slot.

    With in_place=True the given arrays (C-contiguous, writable) are written
    and returned instead of copies.
    """
    k = _c(k)
    v = _c(v)
    if in_place:
        if not (k_cache.flags.c_contiguous and v_cache.flags.c_contiguous and k_cache.flags.writeable
                and v_cache.flags.writeable):
            raise ValueError("in-place write needs C-contiguous, writable caches")
        kc, vc = k_cache, v_cache
    else:
        kc = np.array(k_cache, copy=True, order="C")
        vc = np.array(v_cache, copy=True, order="C")
    sm = _c(slot_mapping, np.int64)
    NB, bs, Hk, D = kc.shape
    token_bytes = Hk * D * kc.itemsize
    assert k.shape[0] == sm.shape[0] and k.dtype == kc.dtype
    n = _load().pa_oracle_reshape_and_cache(_ptr(k), _ptr(v), _ptr(kc), _ptr(vc), _ptr(sm), sm.shape[0],
                                            NB * bs, token_bytes)
    if n < 0:
        raise OracleError("slot outside the pool")
    return kc, vc


def copy_blocks(k_cache, v_cache, pairs):
    """Return copies of (k_cache, v_cache) where block dst of each (src, dst) pair, in order, copies block src."""
    kc = np.array(k_cache, copy=True, order="C")
    vc = np.array(v_cache, copy=True, order="C")
    pr = _c(pairs, np.int64).reshape(-1, 2)
    NB = kc.shape[0]
    bb = kc[0].nbytes
    rc = _load().pa_oracle_copy_blocks(_ptr(kc), _ptr(vc), _ptr(pr), pr.shape[0], NB, bb)
    if rc:
        raise OracleError("block index outside the pool")
    return kc, vc


def swap_blocks(dst, src, pairs):
    """Return a copy of dst where block dst_id of each (src_id, dst_id) pair copies block src_id of src."""
    d = np.array(dst, copy=True, order="C")
    sr = _c(src)
    pr = _c(pairs, np.int64).reshape(-1, 2)
    assert d.dtype == sr.dtype and d.shape[1:] == sr.shape[1:]
    rc = _load().pa_oracle_swap_blocks(_ptr(d), _ptr(sr), _ptr(pr), pr.shape[0], sr.shape[0], d.shape[0], d[0].nbytes)
    if rc:
        raise OracleError("block index outside a pool")
    return d


def e4m3_decode(code: int) -> float:
    return float(_load().pa_oracle_e4m3_decode(int(code) & 0xFF))


def e4m3_encode(x: float) -> int:
    """Nearest E4M3 code of a float32 value (ties to even, saturating at 448)."""
    return int(_load().pa_oracle_e4m3_encode(float(np.float32(x))))


def reshape_and_cache_fp8(k, v, k_cache, v_cache, slot_mapping, k_inv_scale: float, v_inv_scale: float):
    """Quantize bf16 rows (uint16 bits) into copies of the uint8 E4M3 caches at their slots."""
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    kc = np.array(k_cache, copy=True, order="C")
    vc = np.array(v_cache, copy=True, order="C")
    assert kc.dtype == np.uint8
    sm = _c(slot_mapping, np.int64)
    NB, bs, Hk, D = kc.shape
    n = _load().pa_oracle_reshape_and_cache_fp8(_ptr(k), _ptr(v), _ptr(kc), _ptr(vc), _ptr(sm), sm.shape[0], NB * bs,
                                                Hk * D, float(np.float32(k_inv_scale)), float(np.float32(v_inv_scale)))
    if n < 0:
        raise OracleError("slot outside the pool")
    return kc, vc


def decode_fp8(q, k_cache, v_cache, k_scale: float, v_scale: float, block_tables, context_lens, scale: float,
               num_threads: int = 0):
    """Decode over E4M3 caches (uint8 codes): K, V = code value times k_scale, v_scale."""
    q = _c(q)
    k_cache = _c(k_cache, np.uint8)
    v_cache = _c(v_cache, np.uint8)
    bt = _c(block_tables, np.int32)
    cl = _c(context_lens, np.int32)
    B, H, D = q.shape
    NB, bs, Hk, D2 = k_cache.shape
    assert D == D2
    out = np.zeros((B, H, D), np.float64)
    rc = _load().pa_oracle_decode_fp8(_ptr(out), _ptr(q), _dtype_code(q), _ptr(k_cache), _ptr(v_cache),
                                      float(k_scale), float(v_scale), _ptr(bt), bt.shape[1], _ptr(cl), B, H, Hk, D,
                                      bs, NB, float(scale), int(num_threads))
    if rc:
        raise OracleError("decode failed (%d)" % rc)
    return out


def prefill_fp8(q, k_cache, v_cache, k_scale: float, v_scale: float, block_tables, cu_q_lens, context_lens,
                scale: float, rows=None, num_threads: int = 0):
    """Causal chunk attention over E4M3 caches (uint8 codes): K, V = code value times k_scale, v_scale.
    out [T or len(rows), H, D] fp64."""
    q = _c(q)
    k_cache = _c(k_cache, np.uint8)
    v_cache = _c(v_cache, np.uint8)
    bt = _c(block_tables, np.int32)
    cu = _c(cu_q_lens, np.int32)
    cl = _c(context_lens, np.int32)
    T, H, D = q.shape
    NB, bs, Hk, D2 = k_cache.shape
    B = cl.shape[0]
    assert D == D2 and cu.shape[0] == B + 1 and int(cu[-1]) == T and bt.shape[0] == B
    if rows is None:
        n_rows, rows_p = T, None
    else:
        rows_arr = _c(rows, np.int32)
        n_rows, rows_p = rows_arr.shape[0], _ptr(rows_arr)
    out = np.zeros((n_rows, H, D), np.float64)
    rc = _load().pa_oracle_prefill_fp8(_ptr(out), _ptr(q), _dtype_code(q), _ptr(k_cache), _ptr(v_cache),
                                       float(k_scale), float(v_scale), _ptr(bt), bt.shape[1], _ptr(cu), _ptr(cl), B, H,
                                       Hk, D, bs, NB, float(scale), rows_p, n_rows, int(num_threads))
    if rc:
        raise OracleError("prefill failed (%d)" % rc)
    return out
