"""B200 (sm_100a) paged KV cache: PagedAttention decode, cache append, CoW.

A thin binding over the C ABI of ``libpaged_kv.so`` (include/paged_kv.h):
argument checks and marshalling only; every step runs in the library's CUDA
kernels or its C++ host bookkeeping.  PyTorch supplies device memory and
streams.  Importing this package fails loudly if the library is not built.

Layouts: pools fp16 [num_blocks][Hkv][block_size][D]; q / out fp16
[B][q_len][Hq][D] ([B][Hq][D] accepted for decode); block_tables int32
[B][max_blocks]; context_lens int32 [B]; slot_mapping int64 [T].
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import numpy as np
import torch

from . import _abi
from ._abi import KVError, check

__all__ = ["KVPool", "KVError", "pool_bytes", "paged_kv_append", "paged_kv_copy_blocks",
           "workspace_size", "paged_decode_attention", "paged_verify_attention",
           "paged_attention", "paged_prefill_attention", "paged_kv_swap_out", "paged_kv_swap_in",
           "swap_staging_bytes", "paged_kv_k_scales", "paged_kv_append_q8k", "paged_attention_q8k",
           "paged_kv_copy_blocks_q8k",
           "device_error", "lib"]

_L = _abi.load()


def lib() -> ctypes.CDLL:
    return _L


def _stream(device: torch.device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, device=None) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")


def _i32p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


# ---------------------------------------------------------------------------
# sizing and host bookkeeping

def _cfg(num_blocks, block_size, num_kv_heads, head_dim, num_layers=1, dtype_bytes=2):
    return _abi.KvPoolConfig(num_blocks, block_size, num_kv_heads, head_dim, num_layers,
                             dtype_bytes)


def pool_bytes(num_blocks, block_size, num_kv_heads, head_dim, num_layers=1, dtype_bytes=2):
    """(per-layer K+V bytes, total bytes) of a pool."""
    per, tot = ctypes.c_uint64(), ctypes.c_uint64()
    c = _cfg(num_blocks, block_size, num_kv_heads, head_dim, num_layers, dtype_bytes)
    check(_L.kv_pool_bytes(ctypes.byref(c), ctypes.byref(per), ctypes.byref(tot)), "kv_pool_bytes")
    return per.value, tot.value


class KVPool:
    """Refcounted block pool with copy-on-write (host bookkeeping, C++)."""

    def __init__(self, num_blocks: int, block_size: int, num_kv_heads: int = 1, head_dim: int = 128,
                 num_layers: int = 1, order: Optional[Sequence[int]] = None):
        c = _cfg(num_blocks, block_size, num_kv_heads, head_dim, num_layers)
        h = ctypes.c_void_p()
        arr = None
        if order is not None:
            arr = np.ascontiguousarray(order, dtype=np.int32)
            if arr.shape != (num_blocks,):
                raise ValueError("order must list every block once")
        check(_L.kv_pool_create(ctypes.byref(c), _i32p(arr) if arr is not None else None,
                                ctypes.byref(h)), "kv_pool_create")
        self._h = h
        self._lib = _L  # kept so close() still works during interpreter shutdown
        self.num_blocks = num_blocks
        self.block_size = block_size

    def close(self):
        if getattr(self, "_h", None):
            self._lib.kv_pool_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    def num_free(self) -> int:
        n = ctypes.c_int32()
        check(_L.kv_pool_num_free(self._h, ctypes.byref(n)), "kv_pool_num_free")
        return n.value

    def alloc(self, n: int) -> list:
        ids = np.zeros(max(n, 1), np.int32)
        check(_L.block_alloc(self._h, n, _i32p(ids)), "block_alloc")
        return ids[:n].tolist()

    def free(self, ids) -> None:
        a = np.ascontiguousarray(ids, dtype=np.int32)
        check(_L.block_free(self._h, _i32p(a), a.size), "block_free")

    def fork(self, ids) -> None:
        a = np.ascontiguousarray(ids, dtype=np.int32)
        check(_L.block_fork(self._h, _i32p(a), a.size), "block_fork")

    def refcount(self, i: int) -> int:
        rc = ctypes.c_int32()
        check(_L.block_refcount(self._h, i, ctypes.byref(rc)), "block_refcount")
        return rc.value

    def reserve_slot(self, table: np.ndarray, n_blocks: int, ctx_len: int):
        """Reserve the slot of token ``ctx_len``; ``table`` (int32, capacity =
        its length) is updated in place.  Returns (slot, n_blocks, cow_src, cow_dst)."""
        assert table.dtype == np.int32 and table.flags["C_CONTIGUOUS"]
        nb = ctypes.c_int32(n_blocks)
        slot = ctypes.c_int64()
        src, dst = ctypes.c_int32(), ctypes.c_int32()
        check(_L.kv_seq_reserve_slot(self._h, _i32p(table), table.size, ctypes.byref(nb), ctx_len,
                                     ctypes.byref(slot), ctypes.byref(src), ctypes.byref(dst)),
              "kv_seq_reserve_slot")
        return slot.value, nb.value, src.value, dst.value

    def reserve_slots(self, tables: np.ndarray, n_blocks: np.ndarray, ctx_lens: np.ndarray):
        """Batched reserve_slot over B sequences (tables [B][cap] and n_blocks
        [B] updated in place).  Returns (slots int64 [B], cow pairs int32 [k][2])."""
        assert tables.dtype == np.int32 and tables.flags["C_CONTIGUOUS"] and tables.ndim == 2
        assert n_blocks.dtype == np.int32 and n_blocks.flags["C_CONTIGUOUS"]
        B, cap = tables.shape
        cl = np.ascontiguousarray(ctx_lens, dtype=np.int32)
        slots = np.zeros(B, np.int64)
        pairs = np.zeros((max(B, 1), 2), np.int32)
        ncow, ndone = ctypes.c_int32(), ctypes.c_int32()
        check(_L.kv_batch_reserve_slots(self._h, B, _i32p(tables), cap, _i32p(n_blocks), _i32p(cl),
                                        slots.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                        _i32p(pairs), ctypes.byref(ncow), ctypes.byref(ndone)),
              "kv_batch_reserve_slots")
        return slots, pairs[:ncow.value].copy()

    def beam_reorder(self, tables: np.ndarray, n_blocks: np.ndarray, parents):
        """One beam-search step: new beam i continues old beam parents[i].
        Returns (new_tables int32 [n_new][cap], new_n_blocks int32 [n_new])."""
        assert tables.dtype == np.int32 and tables.flags["C_CONTIGUOUS"] and tables.ndim == 2
        nb = np.ascontiguousarray(n_blocks, dtype=np.int32)
        par = np.ascontiguousarray(parents, dtype=np.int32)
        B, cap = tables.shape
        new = np.full((max(par.size, 1), cap), -1, np.int32)
        new_nb = np.zeros(max(par.size, 1), np.int32)
        check(_L.kv_beam_reorder(self._h, _i32p(tables), _i32p(nb), B, cap, _i32p(par), par.size,
                                 _i32p(new), _i32p(new_nb)), "kv_beam_reorder")
        return new[:par.size].copy(), new_nb[:par.size].copy()

    # -- prefix cache --------------------------------------------------------
    def prefix_match(self, tokens) -> list:
        """Cached blocks holding the longest cached prefix of ``tokens`` (one
        reference added to each, for the caller)."""
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        cap = t.size // self.block_size
        out = np.zeros(max(cap, 1), np.int32)
        n = ctypes.c_int32()
        check(_L.kv_prefix_match(self._h, _i32p(t), t.size, _i32p(out), cap, ctypes.byref(n)),
              "kv_prefix_match")
        return out[:n.value].tolist()

    def prefix_register(self, tokens, table) -> int:
        """Cache the full blocks of a request; returns how many leading blocks
        of ``table`` are now cached under this prefix."""
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        b = np.ascontiguousarray(table, dtype=np.int32)
        n = ctypes.c_int32()
        check(_L.kv_prefix_register(self._h, _i32p(t), t.size, _i32p(b), b.size, ctypes.byref(n)),
              "kv_prefix_register")
        return n.value

    def prefix_evict(self, n: int) -> list:
        ids = np.zeros(max(n, 1), np.int32)
        k = ctypes.c_int32()
        check(_L.kv_prefix_evict(self._h, n, _i32p(ids), ctypes.byref(k)), "kv_prefix_evict")
        return ids[:k.value].tolist()

    def num_cached(self) -> int:
        n = ctypes.c_int32()
        check(_L.kv_prefix_num_cached(self._h, ctypes.byref(n)), "kv_prefix_num_cached")
        return n.value


# ---------------------------------------------------------------------------
# device calls

def paged_kv_append(k_new: torch.Tensor, v_new: torch.Tensor, slot_mapping: torch.Tensor,
                    k_pool: torch.Tensor, v_pool: torch.Tensor) -> None:
    dev = k_pool.device
    for t, n in ((k_pool, "k_pool"), (v_pool, "v_pool"), (k_new, "k_new"), (v_new, "v_new")):
        _need(t, n, torch.float16, dev)
    _need(slot_mapping, "slot_mapping", torch.int64, dev)
    nb, Hkv, bs, D = k_pool.shape
    T = slot_mapping.numel()
    if k_new.numel() != T * Hkv * D or v_new.numel() != T * Hkv * D or v_pool.shape != k_pool.shape:
        raise ValueError("paged_kv_append: shape mismatch")
    check(_L.paged_kv_append(k_new.data_ptr(), v_new.data_ptr(), slot_mapping.data_ptr(),
                             k_pool.data_ptr(), v_pool.data_ptr(), T, Hkv, D, bs, nb, _stream(dev)),
          "paged_kv_append")


def paged_kv_copy_blocks(k_pool: torch.Tensor, v_pool: torch.Tensor, pairs: torch.Tensor) -> None:
    dev = k_pool.device
    _need(k_pool, "k_pool", torch.float16, dev)
    _need(v_pool, "v_pool", torch.float16, dev)
    _need(pairs, "pairs", torch.int32, dev)
    nb, Hkv, bs, D = k_pool.shape
    n = pairs.numel() // 2
    check(_L.paged_kv_copy_blocks(k_pool.data_ptr(), v_pool.data_ptr(), pairs.data_ptr(), n, Hkv, D,
                                  bs, nb, _stream(dev)), "paged_kv_copy_blocks")


def swap_staging_bytes(k_pool: torch.Tensor, n: int) -> int:
    """Bytes of the staging (and host) buffer of a swap of n blocks."""
    _, Hkv, bs, D = k_pool.shape
    return 2 * n * Hkv * bs * D * 2


def paged_kv_swap_out(k_pool: torch.Tensor, v_pool: torch.Tensor, block_ids: torch.Tensor,
                      staging: torch.Tensor, host: Optional[torch.Tensor] = None) -> None:
    """K and V of ``block_ids`` (device int32) -> ``staging`` (device, uint8 or
    fp16) -> ``host`` (pinned CPU tensor of the same byte size, optional)."""
    dev = k_pool.device
    _need(k_pool, "k_pool", torch.float16, dev)
    _need(v_pool, "v_pool", torch.float16, dev)
    _need(block_ids, "block_ids", torch.int32, dev)
    nb, Hkv, bs, D = k_pool.shape
    n = block_ids.numel()
    _swap_buffers(staging, host, dev, swap_staging_bytes(k_pool, n))
    check(_L.paged_kv_swap_out(k_pool.data_ptr(), v_pool.data_ptr(), block_ids.data_ptr(), n,
                               staging.data_ptr(), host.data_ptr() if host is not None else None, Hkv,
                               D, bs, nb, _stream(dev)), "paged_kv_swap_out")


def paged_kv_swap_in(k_pool: torch.Tensor, v_pool: torch.Tensor, block_ids: torch.Tensor,
                     staging: torch.Tensor, host: Optional[torch.Tensor] = None) -> None:
    """``host`` (optional) -> ``staging`` -> K and V of ``block_ids``."""
    dev = k_pool.device
    _need(k_pool, "k_pool", torch.float16, dev)
    _need(v_pool, "v_pool", torch.float16, dev)
    _need(block_ids, "block_ids", torch.int32, dev)
    nb, Hkv, bs, D = k_pool.shape
    n = block_ids.numel()
    _swap_buffers(staging, host, dev, swap_staging_bytes(k_pool, n))
    check(_L.paged_kv_swap_in(k_pool.data_ptr(), v_pool.data_ptr(), block_ids.data_ptr(), n,
                              staging.data_ptr(), host.data_ptr() if host is not None else None, Hkv,
                              D, bs, nb, _stream(dev)), "paged_kv_swap_in")


def _swap_buffers(staging, host, dev, nbytes):
    if staging.device != dev or not staging.is_contiguous():
        raise ValueError("staging must be a contiguous tensor on the pools' device")
    if staging.numel() * staging.element_size() < nbytes:
        raise ValueError(f"staging holds fewer than {nbytes} bytes")
    if host is not None:
        if host.device.type != "cpu" or not host.is_contiguous():
            raise ValueError("host must be a contiguous CPU tensor")
        if host.numel() * host.element_size() < nbytes:
            raise ValueError(f"host holds fewer than {nbytes} bytes")


def workspace_size(Hq: int, Hkv: int, q_len: int, head_dim: int, grid_ctas: int = 0) -> int:
    n = ctypes.c_size_t()
    check(_L.paged_attention_workspace_size(Hq, Hkv, q_len, head_dim, grid_ctas, ctypes.byref(n)),
          "paged_attention_workspace_size")
    return n.value


def _attention(q, k_pool, v_pool, block_tables, context_lens, scale, q_len, out, workspace,
               grid_ctas, min_split_blocks, use_pdl, entry, seg_cost_blocks=0, k_scales=None,
               producer_wait_ns=0, consumer=0):
    dev = k_pool.device
    _need(k_pool, "k_pool", torch.int8 if entry == "q8k" else torch.float16, dev)
    for t, n in ((q, "q"), (v_pool, "v_pool")):
        _need(t, n, torch.float16, dev)
    if entry == "q8k":
        _need(k_scales, "k_scales", torch.float32, dev)
        if tuple(k_scales.shape) != (k_pool.shape[1], k_pool.shape[3]):
            raise ValueError("k_scales must be [Hkv][D]")
    _need(block_tables, "block_tables", torch.int32, dev)
    _need(context_lens, "context_lens", torch.int32, dev)
    nb, Hkv, bs, D = k_pool.shape
    B = context_lens.numel()
    Hq = q.shape[-2]
    if q.shape[-1] != D or q.numel() != B * q_len * Hq * D:
        raise ValueError("q must be [B][q_len][Hq][D]")
    if block_tables.dim() != 2 or block_tables.shape[0] != B:
        raise ValueError("block_tables must be [B][max_blocks]")
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.float16, dev)
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    if workspace is None:  # (a caller's workspace is size-checked by the library)
        workspace = torch.empty(workspace_size(Hq, Hkv, q_len, D, grid_ctas), dtype=torch.uint8,
                                device=dev)
    _need(workspace, "workspace", torch.uint8, dev)
    mb = block_tables.shape[1]
    args = (q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(), block_tables.data_ptr(), mb,
            context_lens.data_ptr())
    tail = (float(scale), out.data_ptr(), B, Hq, Hkv, D, bs, nb, workspace.data_ptr(),
            workspace.numel())
    if entry == "decode":
        rc = _L.paged_decode_attention(*args, *tail, _stream(dev))
    elif entry == "verify":
        rc = _L.paged_verify_attention(*args, q_len, *tail, _stream(dev))
    elif entry == "q8k":
        q8 = (q.data_ptr(), k_pool.data_ptr(), k_scales.data_ptr(), v_pool.data_ptr(),
              block_tables.data_ptr(), mb, context_lens.data_ptr(), q_len)
        if grid_ctas or min_split_blocks or use_pdl or seg_cost_blocks or producer_wait_ns or consumer:
            o = _abi.PagedAttentionOpts(grid_ctas, min_split_blocks, use_pdl, seg_cost_blocks,
                                        producer_wait_ns, consumer)
            rc = _L.paged_attention_q8k_ex(*q8, *tail, ctypes.byref(o), _stream(dev))
        else:
            rc = _L.paged_attention_q8k(*q8, *tail, _stream(dev))
    else:
        o = _abi.PagedAttentionOpts(grid_ctas, min_split_blocks, use_pdl, seg_cost_blocks,
                                    producer_wait_ns, consumer)
        rc = _L.paged_attention_ex(*args, q_len, *tail, ctypes.byref(o), _stream(dev))
    check(rc, f"paged attention ({entry})")
    return out


def paged_kv_k_scales(k: torch.Tensor) -> torch.Tensor:
    """Per-(KV head, channel) scales max|k| / 127 of calibration keys
    k [T][Hkv][D] fp16 (device) -> fp32 [Hkv][D]."""
    dev = k.device
    _need(k, "k", torch.float16, dev)
    T, Hkv, D = k.shape
    out = torch.empty((Hkv, D), dtype=torch.float32, device=dev)
    check(_L.paged_kv_k_scales(k.data_ptr(), T, Hkv, D, out.data_ptr(), _stream(dev)),
          "paged_kv_k_scales")
    return out


def paged_kv_append_q8k(k_new: torch.Tensor, v_new: torch.Tensor, slot_mapping: torch.Tensor,
                        k_scales: torch.Tensor, kq_pool: torch.Tensor, v_pool: torch.Tensor) -> None:
    """Append with K quantised to int8 codes (per-channel scales), V as fp16."""
    dev = v_pool.device
    _need(kq_pool, "kq_pool", torch.int8, dev)
    for t, n in ((v_pool, "v_pool"), (k_new, "k_new"), (v_new, "v_new")):
        _need(t, n, torch.float16, dev)
    _need(k_scales, "k_scales", torch.float32, dev)
    _need(slot_mapping, "slot_mapping", torch.int64, dev)
    nb, Hkv, bs, D = kq_pool.shape
    if tuple(v_pool.shape) != (nb, Hkv, bs, D) or tuple(k_scales.shape) != (Hkv, D):
        raise ValueError("pool / scale shapes disagree")
    T = slot_mapping.numel()
    check(_L.paged_kv_append_q8k(k_new.data_ptr(), v_new.data_ptr(), slot_mapping.data_ptr(),
                                 k_scales.data_ptr(), kq_pool.data_ptr(), v_pool.data_ptr(), T, Hkv,
                                 D, bs, nb, _stream(dev)), "paged_kv_append_q8k")


def paged_kv_copy_blocks_q8k(kq_pool: torch.Tensor, v_pool: torch.Tensor, pairs: torch.Tensor) -> None:
    """Copy-on-write block copies for an int8 K pool and its fp16 V pool."""
    dev = v_pool.device
    _need(kq_pool, "kq_pool", torch.int8, dev)
    _need(v_pool, "v_pool", torch.float16, dev)
    _need(pairs, "pairs", torch.int32, dev)
    nb, Hkv, bs, D = kq_pool.shape
    check(_L.paged_kv_copy_blocks_q8k(kq_pool.data_ptr(), v_pool.data_ptr(), pairs.data_ptr(),
                                      pairs.numel() // 2, Hkv, D, bs, nb, _stream(dev)),
          "paged_kv_copy_blocks_q8k")


def paged_attention_q8k(q, kq_pool, k_scales, v_pool, block_tables, context_lens, scale, q_len=1,
                        out=None, workspace=None, grid_ctas=0, min_split_blocks=0, use_pdl=0,
                        seg_cost_blocks=0, producer_wait_ns=0, consumer=0):
    """Decode (q_len = 1) or causal verify attention over an int8 K pool
    (launch knobs as in paged_attention)."""
    return _attention(q, kq_pool, v_pool, block_tables, context_lens, scale, q_len, out, workspace,
                      grid_ctas, min_split_blocks, use_pdl, "q8k", seg_cost_blocks, k_scales=k_scales,
                      producer_wait_ns=producer_wait_ns, consumer=consumer)


def paged_decode_attention(q, k_pool, v_pool, block_tables, context_lens, scale, out=None,
                           workspace=None):
    """out[s][h] = softmax(scale q K^T) V over the first context_lens[s] tokens."""
    return _attention(q, k_pool, v_pool, block_tables, context_lens, scale, 1, out, workspace,
                      0, 0, 0, "decode")


def paged_verify_attention(q, k_pool, v_pool, block_tables, context_lens, scale, q_len, out=None,
                           workspace=None):
    """Causal verify window: row j sees tokens 0 .. context_lens[s] - q_len + j."""
    return _attention(q, k_pool, v_pool, block_tables, context_lens, scale, q_len, out, workspace,
                      0, 0, 0, "verify")


def paged_attention(q, k_pool, v_pool, block_tables, context_lens, scale, q_len=1, out=None,
                    workspace=None, grid_ctas=0, min_split_blocks=0, use_pdl=0, seg_cost_blocks=0,
                    producer_wait_ns=0, consumer=0):
    """Decode / verify with launch knobs (grid size, smallest split, PDL,
    per-segment cost used to balance CTAs, the loading warp's wait limit for
    failure-detection tests, the compute path for several query rows per KV
    head: 1 warp-level MMAs, 2 tcgen05 with tensor-memory accumulators, 0
    default)."""
    return _attention(q, k_pool, v_pool, block_tables, context_lens, scale, q_len, out, workspace,
                      grid_ctas, min_split_blocks, use_pdl, "ex", seg_cost_blocks,
                      producer_wait_ns=producer_wait_ns, consumer=consumer)


def paged_prefill_attention(q, k_pool, v_pool, block_tables, context_lens, scale, q_len,
                            out=None, producer_wait_ns=0):
    """Causal chunked prefill over the paged cache (tensor cores): row j of
    sequence s sees tokens 0 .. context_lens[s] - q_len + j.  producer_wait_ns:
    the loading warp's wait limit, for failure-detection tests."""
    dev = k_pool.device
    for t, n in ((q, "q"), (k_pool, "k_pool"), (v_pool, "v_pool")):
        _need(t, n, torch.float16, dev)
    _need(block_tables, "block_tables", torch.int32, dev)
    _need(context_lens, "context_lens", torch.int32, dev)
    nb, Hkv, bs, D = k_pool.shape
    B = context_lens.numel()
    Hq = q.shape[-2]
    if q.shape[-1] != D or q.numel() != B * q_len * Hq * D:
        raise ValueError("q must be [B][q_len][Hq][D]")
    if block_tables.dim() != 2 or block_tables.shape[0] != B:
        raise ValueError("block_tables must be [B][max_blocks]")
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.float16, dev)
    args = (q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(), block_tables.data_ptr(),
            block_tables.shape[1], context_lens.data_ptr(), q_len, float(scale), out.data_ptr(),
            B, Hq, Hkv, D, bs, nb)
    if producer_wait_ns:
        o = _abi.PagedAttentionOpts(0, 0, 0, 0, producer_wait_ns)
        check(_L.paged_prefill_attention_ex(*args, ctypes.byref(o), _stream(dev)),
              "paged_prefill_attention_ex")
    else:
        check(_L.paged_prefill_attention(*args, _stream(dev)), "paged_prefill_attention")
    return out


def device_error(reset: bool = True, device=None) -> int:
    """Synchronise the current stream and return (optionally clear) the
    device error word (bits KV_DEV_*)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    w = ctypes.c_int32()
    check(_L.kv_device_error(ctypes.byref(w), 1 if reset else 0, _stream(dev)), "kv_device_error")
    return w.value
