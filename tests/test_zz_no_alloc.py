"""The allocation-free decode entry point (needs a B200).

paged_decode_attention_static_ws serves callers that cannot allocate device
memory themselves: it takes no workspace and uses scratch built into the
library.  Its output must match paged_decode_attention's (same inputs,
caller-allocated workspace) within the attention tolerance, on two calls in a
row (the second call meets the scratch as the first call left it).

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from paged_helpers import ATOL, RTOL
from workloads import make_workload

pytestmark = pytest.mark.gpu


def _call_static(L, wl, bt, cl, out):
    nb, Hkv, bs, D = wl.k_pool.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.paged_decode_attention_static_ws(
        wl.q.data_ptr(), wl.k_pool.data_ptr(), wl.v_pool.data_ptr(), bt.data_ptr(), bt.shape[1],
        cl.data_ptr(), ctypes.c_float(wl.scale), out.data_ptr(), wl.B, wl.q.shape[-2], Hkv, D, bs,
        nb, stream)


@pytest.mark.parametrize("name,kw", [("llama70b_gqa", {"B": 24, "max_len": 3000}),
                                     ("llama7b_mha", {"B": 8, "max_len": 2000})])
def test_static_scratch_matches_workspace_entry(name, kw):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import paged_kv_cache_371_b200 as pkv
    L = pkv.lib()
    wl = make_workload(name, "cuda", **kw)
    bt = torch.as_tensor(wl.block_tables, device="cuda")
    cl = torch.as_tensor(wl.lens, device="cuda")
    ref = pkv.paged_decode_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale)
    torch.cuda.synchronize()
    for call in range(2):
        out = torch.full_like(wl.q, float("nan"))
        rc = _call_static(L, wl, bt, cl, out)
        assert rc == 0, L.kv_last_error_string()
        torch.cuda.synchronize()
        assert pkv.device_error() == 0
        a = out.float().cpu().numpy()
        b = ref.float().cpu().numpy()
        assert np.isfinite(a).all(), f"call {call}: non-finite output"
        assert (np.abs(a - b) <= ATOL + RTOL * np.abs(b)).all(), f"call {call}: mismatch"


def test_static_scratch_rejects_bad_shapes_without_launch():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import paged_kv_cache_371_b200 as pkv
    L = pkv.lib()
    wl = make_workload("tiny", "cuda")
    bt = torch.as_tensor(wl.block_tables, device="cuda")
    cl = torch.as_tensor(wl.lens, device="cuda")
    out = torch.empty_like(wl.q)
    nb, Hkv, bs, D = wl.k_pool.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # 64 query heads per KV head exceeds what the kernels serve: refused up front
    rc = L.paged_decode_attention_static_ws(
        wl.q.data_ptr(), wl.k_pool.data_ptr(), wl.v_pool.data_ptr(), bt.data_ptr(), bt.shape[1],
        cl.data_ptr(), ctypes.c_float(wl.scale), out.data_ptr(), wl.B, 64, 1, D, bs, nb, stream)
    assert rc == pkv._abi.KV_ERR_INVALID
