"""Paged-KV oracle (fp64, CPU) — test infrastructure.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library and its Python binding
never import it, and it never imports them.

The arithmetic lives in ``paged_oracle.c`` (plain C, fp64) and the host
bookkeeping policy in ``block_spec.py`` (plain Python).  This module only
marshals numpy arrays into the C functions.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib(path: str | None = None) -> ctypes.CDLL:
    """Load (building first if needed) the oracle shared object."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(_build.build()))
    return _lib


def _bind(L: ctypes.CDLL) -> ctypes.CDLL:
    P = ctypes.c_void_p
    i32 = ctypes.c_int32
    u64 = ctypes.c_uint64
    L.oracle_half_to_double.argtypes = [ctypes.c_uint16]
    L.oracle_half_to_double.restype = ctypes.c_double
    L.oracle_num_threads.restype = ctypes.c_int
    L.oracle_set_num_threads.argtypes = [ctypes.c_int]
    L.oracle_kv_cache_bytes.argtypes = [u64] * 6
    L.oracle_kv_cache_bytes.restype = u64
    L.oracle_pool_bytes_per_layer.argtypes = [u64] * 5
    L.oracle_pool_bytes_per_layer.restype = u64
    L.oracle_paged_attention.argtypes = [P, P, P, P, i32, P, i32, i32, i32, i32, i32, i32, i32,
                                         ctypes.c_double, P]
    L.oracle_paged_attention.restype = ctypes.c_int
    L.oracle_append.argtypes = [P, P, P, i32, i32, i32, i32, i32, P, P]
    L.oracle_append.restype = ctypes.c_int
    L.oracle_copy_blocks.argtypes = [P, i32, i32, i32, i32, i32, P, P]
    L.oracle_copy_blocks.restype = ctypes.c_int
    L.oracle_k_scales.argtypes = [P, ctypes.c_int64, i32, i32, P]
    L.oracle_k_scales.restype = ctypes.c_int
    L.oracle_append_q8k.argtypes = [P, P, P, i32, i32, i32, i32, i32, P, P, P]
    L.oracle_append_q8k.restype = ctypes.c_int
    L.oracle_paged_attention_q8k.argtypes = [P, P, P, P, P, i32, P, i32, i32, i32, i32, i32, i32,
                                             i32, ctypes.c_double, P]
    L.oracle_paged_attention_q8k.restype = ctypes.c_int
    return L


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _as_u16(a: np.ndarray) -> np.ndarray:
    """fp16 array -> its raw 16-bit patterns (no value conversion)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    assert a.dtype == np.uint16
    return a


def half_to_double(h: int, L: ctypes.CDLL | None = None) -> float:
    return (L or lib()).oracle_half_to_double(int(h) & 0xFFFF)


def num_threads() -> int:
    return lib().oracle_num_threads()


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))


def kv_cache_bytes(layers, heads, head_dim, seq_len, batch, dtype_bytes) -> int:
    return int(lib().oracle_kv_cache_bytes(layers, heads, head_dim, seq_len, batch, dtype_bytes))


def pool_bytes_per_layer(num_blocks, block_size, num_kv_heads, head_dim, dtype_bytes) -> int:
    return int(lib().oracle_pool_bytes_per_layer(num_blocks, block_size, num_kv_heads, head_dim,
                                                 dtype_bytes))


def paged_attention(q, k_pool, v_pool, block_tables, context_lens, *, scale, q_len=1,
                    L: ctypes.CDLL | None = None) -> np.ndarray:
    """Exact attention over the paged cache, fp64.

    q: fp16 [B][q_len][Hq][D] (or [B][Hq][D] when q_len == 1);
    k_pool / v_pool: fp16 [num_blocks][Hkv][bs][D];
    block_tables: int32 [B][max_blocks]; context_lens: int32 [B].
    Returns fp64 with q's shape.
    """
    L = L or lib()
    q16 = _as_u16(q)
    k16 = _as_u16(k_pool)
    v16 = _as_u16(v_pool)
    nb, Hkv, bs, D = k16.shape
    assert v16.shape == k16.shape
    B = int(context_lens.shape[0])
    Hq = q16.shape[-2]
    assert q16.shape[-1] == D and q16.size == B * q_len * Hq * D
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    if bt.ndim == 1:
        bt = bt.reshape(B, -1)
    out = np.zeros(q16.shape, dtype=np.float64)
    rc = L.oracle_paged_attention(_ptr(q16), _ptr(k16), _ptr(v16), _ptr(bt), bt.shape[1],
                                  _ptr(cl), B, q_len, Hq, Hkv, D, bs, nb, float(scale),
                                  _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_paged_attention rejected its inputs (code {rc})")
    return out


def append(k_pool, v_pool, k_new, v_new, slot_mapping, L: ctypes.CDLL | None = None):
    """Return copies of the pools with the new tokens written into their slots."""
    L = L or lib()
    k16 = _as_u16(k_pool).copy()
    v16 = _as_u16(v_pool).copy()
    nb, Hkv, bs, D = k16.shape
    kn = _as_u16(k_new)
    vn = _as_u16(v_new)
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    T = int(sm.shape[0])
    assert kn.size == T * Hkv * D and vn.size == T * Hkv * D
    rc = L.oracle_append(_ptr(kn), _ptr(vn), _ptr(sm), T, Hkv, D, bs, nb, _ptr(k16), _ptr(v16))
    if rc != 0:
        raise ValueError(f"oracle_append rejected its inputs (code {rc})")
    return k16.view(np.float16), v16.view(np.float16)


def copy_blocks(k_pool, v_pool, pairs, L: ctypes.CDLL | None = None):
    """Return copies of the pools after the (src, dst) whole-block copies."""
    L = L or lib()
    k16 = _as_u16(k_pool).copy()
    v16 = _as_u16(v_pool).copy()
    nb, Hkv, bs, D = k16.shape
    pr = np.ascontiguousarray(pairs, dtype=np.int32).reshape(-1)
    rc = L.oracle_copy_blocks(_ptr(pr), pr.size // 2, Hkv, D, bs, nb, _ptr(k16), _ptr(v16))
    if rc != 0:
        raise ValueError(f"oracle_copy_blocks rejected its inputs (code {rc})")
    return k16.view(np.float16), v16.view(np.float16)


# -- quantised K pool (int8 codes, one fp32 scale per KV head and channel) --
def k_scales(k, L: ctypes.CDLL | None = None) -> np.ndarray:
    """Per-(KV head, channel) scales max|k| / 127 of calibration keys
    k: fp16 [T][Hkv][D] -> fp32 [Hkv][D]."""
    L = L or lib()
    k16 = _as_u16(k)
    T, Hkv, D = k16.shape
    out = np.zeros((Hkv, D), np.float32)
    rc = L.oracle_k_scales(_ptr(k16), T, Hkv, D, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_k_scales rejected its inputs (code {rc})")
    return out


def append_q8k(kq_pool, v_pool, k_new, v_new, slot_mapping, scales, L: ctypes.CDLL | None = None):
    """Return copies of the code pool (int8) and V pool with the new tokens
    written: K quantised with ``scales``, V as is."""
    L = L or lib()
    k8 = np.ascontiguousarray(kq_pool, dtype=np.int8).copy()
    v16 = _as_u16(v_pool).copy()
    nb, Hkv, bs, D = k8.shape
    kn, vn = _as_u16(k_new), _as_u16(v_new)
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    sc = np.ascontiguousarray(scales, dtype=np.float32)
    T = int(sm.shape[0])
    assert kn.size == T * Hkv * D and vn.size == T * Hkv * D and sc.shape == (Hkv, D)
    rc = L.oracle_append_q8k(_ptr(kn), _ptr(vn), _ptr(sm), T, Hkv, D, bs, nb, _ptr(sc), _ptr(k8),
                             _ptr(v16))
    if rc != 0:
        raise ValueError(f"oracle_append_q8k rejected its inputs (code {rc})")
    return k8, v16.view(np.float16)


def paged_attention_q8k(q, kq_pool, scales, v_pool, block_tables, context_lens, *, scale, q_len=1,
                        L: ctypes.CDLL | None = None) -> np.ndarray:
    """Exact attention with K = code * scale (fp64), V fp16; as paged_attention."""
    L = L or lib()
    q16 = _as_u16(q)
    k8 = np.ascontiguousarray(kq_pool, dtype=np.int8)
    v16 = _as_u16(v_pool)
    nb, Hkv, bs, D = k8.shape
    sc = np.ascontiguousarray(scales, dtype=np.float32)
    B = int(context_lens.shape[0])
    Hq = q16.shape[-2]
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    if bt.ndim == 1:
        bt = bt.reshape(B, -1)
    out = np.zeros(q16.shape, dtype=np.float64)
    rc = L.oracle_paged_attention_q8k(_ptr(q16), _ptr(k8), _ptr(sc), _ptr(v16), _ptr(bt), bt.shape[1],
                                      _ptr(cl), B, q_len, Hq, Hkv, D, bs, nb, float(scale), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_paged_attention_q8k rejected its inputs (code {rc})")
    return out

