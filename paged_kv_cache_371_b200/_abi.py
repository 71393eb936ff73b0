"""ctypes view of ``libpaged_kv.so`` (declared in include/paged_kv.h)."""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpaged_kv.so")

KV_OK = 0
KV_ERR_INVALID = 1
KV_ERR_OOM = 2
KV_ERR_DOUBLE_FREE = 3
KV_ERR_CUDA = 4

KV_DEV_BAD_BLOCK = 1
KV_DEV_BAD_SLOT = 2
KV_DEV_TIMEOUT = 4
KV_DEV_BAD_SCALE = 8


class KvPoolConfig(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("num_layers", ctypes.c_int32), ("dtype_bytes", ctypes.c_int32)]


class PagedAttentionOpts(ctypes.Structure):
    _fields_ = [("grid_ctas", ctypes.c_int32), ("min_split_blocks", ctypes.c_int32),
                ("use_pdl", ctypes.c_int32), ("seg_cost_blocks", ctypes.c_int32),
                ("producer_wait_ns", ctypes.c_int32), ("consumer", ctypes.c_int32),
                ("reserved", ctypes.c_int32 * 2)]


_P = ctypes.c_void_p
_i32 = ctypes.c_int32
_PI32 = ctypes.POINTER(ctypes.c_int32)
_PI64 = ctypes.POINTER(ctypes.c_int64)
_sz = ctypes.c_size_t

SIGNATURES = {
    "kv_last_error_string": ([], ctypes.c_char_p),
    "kv_version": ([], ctypes.c_int),
    "kv_pool_bytes": ([ctypes.POINTER(KvPoolConfig), ctypes.POINTER(ctypes.c_uint64),
                       ctypes.POINTER(ctypes.c_uint64)], ctypes.c_int),
    "kv_pool_create": ([ctypes.POINTER(KvPoolConfig), _PI32, ctypes.POINTER(_P)], ctypes.c_int),
    "kv_pool_destroy": ([_P], ctypes.c_int),
    "kv_pool_num_free": ([_P, _PI32], ctypes.c_int),
    "block_alloc": ([_P, _i32, _PI32], ctypes.c_int),
    "block_free": ([_P, _PI32, _i32], ctypes.c_int),
    "block_fork": ([_P, _PI32, _i32], ctypes.c_int),
    "block_refcount": ([_P, _i32, _PI32], ctypes.c_int),
    "kv_seq_reserve_slot": ([_P, _PI32, _i32, _PI32, _i32, _PI64, _PI32, _PI32], ctypes.c_int),
    "kv_batch_reserve_slots": ([_P, _i32, _PI32, _i32, _PI32, _PI32, _PI64, _PI32, _PI32, _PI32],
                               ctypes.c_int),
    "paged_kv_append": ([_P, _P, _P, _P, _P, _i32, _i32, _i32, _i32, _i32, _P], ctypes.c_int),
    "paged_kv_copy_blocks": ([_P, _P, _P, _i32, _i32, _i32, _i32, _i32, _P], ctypes.c_int),
    "paged_attention_workspace_size": ([_i32, _i32, _i32, _i32, _i32, ctypes.POINTER(_sz)],
                                       ctypes.c_int),
    "paged_decode_attention": ([_P, _P, _P, _P, _i32, _P, ctypes.c_float, _P, _i32, _i32, _i32,
                                _i32, _i32, _i32, _P, _sz, _P], ctypes.c_int),
    "paged_verify_attention": ([_P, _P, _P, _P, _i32, _P, _i32, ctypes.c_float, _P, _i32, _i32,
                                _i32, _i32, _i32, _i32, _P, _sz, _P], ctypes.c_int),
    "paged_attention_ex": ([_P, _P, _P, _P, _i32, _P, _i32, ctypes.c_float, _P, _i32, _i32, _i32,
                            _i32, _i32, _i32, _P, _sz, ctypes.POINTER(PagedAttentionOpts), _P],
                           ctypes.c_int),
    "kv_device_error": ([_PI32, _i32, _P], ctypes.c_int),
    "paged_prefill_attention": ([_P, _P, _P, _P, _i32, _P, _i32, ctypes.c_float, _P, _i32, _i32,
                                 _i32, _i32, _i32, _i32, _P], ctypes.c_int),
    "paged_decode_attention_static_ws": ([_P, _P, _P, _P, _i32, _P, ctypes.c_float, _P, _i32,
                                          _i32, _i32, _i32, _i32, _i32, _P], ctypes.c_int),
    "kv_beam_reorder": ([_P, _PI32, _PI32, _i32, _i32, _PI32, _i32, _PI32, _PI32], ctypes.c_int),
    "kv_prefix_match": ([_P, _PI32, _i32, _PI32, _i32, _PI32], ctypes.c_int),
    "kv_prefix_register": ([_P, _PI32, _i32, _PI32, _i32, _PI32], ctypes.c_int),
    "kv_prefix_evict": ([_P, _i32, _PI32, _PI32], ctypes.c_int),
    "kv_prefix_num_cached": ([_P, _PI32], ctypes.c_int),
    "paged_kv_swap_out": ([_P, _P, _P, _i32, _P, _P, _i32, _i32, _i32, _i32, _P], ctypes.c_int),
    "paged_kv_swap_in": ([_P, _P, _P, _i32, _P, _P, _i32, _i32, _i32, _i32, _P], ctypes.c_int),
    "paged_kv_k_scales": ([_P, ctypes.c_int64, _i32, _i32, _P, _P], ctypes.c_int),
    "paged_kv_copy_blocks_q8k": ([_P, _P, _P, _i32, _i32, _i32, _i32, _i32, _P], ctypes.c_int),
    "paged_kv_append_q8k": ([_P, _P, _P, _P, _P, _P, _i32, _i32, _i32, _i32, _i32, _P], ctypes.c_int),
    "paged_attention_q8k": ([_P, _P, _P, _P, _P, _i32, _P, _i32, ctypes.c_float, _P, _i32, _i32, _i32,
                             _i32, _i32, _i32, _P, _sz, _P], ctypes.c_int),
    "paged_prefill_attention_ex": ([_P, _P, _P, _P, _i32, _P, _i32, ctypes.c_float, _P, _i32, _i32,
                                    _i32, _i32, _i32, _i32, ctypes.POINTER(PagedAttentionOpts), _P],
                                   ctypes.c_int),
    "paged_attention_q8k_ex": ([_P, _P, _P, _P, _P, _i32, _P, _i32, ctypes.c_float, _P, _i32, _i32,
                                _i32, _i32, _i32, _i32, _P, _sz, ctypes.POINTER(PagedAttentionOpts),
                                _P], ctypes.c_int),
}


class KVError(RuntimeError):
    def __init__(self, code: int, where: str, text: str):
        super().__init__(f"{where} failed with status {code}: {text}")
        self.code = code


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library; raises ImportError if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python paged_kv_cache_371_b200/build.py` "
            "(there is no fallback implementation)")
    L = ctypes.CDLL(path)
    for name, (args, res) in SIGNATURES.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def check(rc: int, where: str) -> None:
    if rc != KV_OK:
        raise KVError(rc, where, load().kv_last_error_string().decode(errors="replace"))
