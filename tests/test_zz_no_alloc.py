"""The allocation-free decode entry point (needs a B200).

paged_decode_attention_static_ws serves callers that cannot allocate device
memory themselves (their device memory belongs to another allocator, they
receive tensors but no allocation hook, or a cudaMalloc on their hot path is
not allowed): it takes no workspace and keeps its split-context scratch in a
fixed array inside the library.  Each case here first runs a different
workload through it (so the scratch holds another call's leftovers), then the
checked workload twice in a row.  Every checked call must be bit-identical to
paged_decode_attention with a caller workspace (same kernel, same grid, same
fixed merge order) and within the attention tolerance of the fp64 oracle;
each checked shape is asserted to split contexts across CTAs, so the scratch
really carries partial results.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from paged_helpers import assert_close, oracle_subset
from workloads import make_workload

pytestmark = pytest.mark.gpu


def _call_static(L, wl, bt, cl, out):
    nb, Hkv, bs, D = wl.k_pool.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.paged_decode_attention_static_ws(
        wl.q.data_ptr(), wl.k_pool.data_ptr(), wl.v_pool.data_ptr(), bt.data_ptr(), bt.shape[1],
        cl.data_ptr(), ctypes.c_float(wl.scale), out.data_ptr(), wl.B, wl.q.shape[-2], Hkv, D, bs,
        nb, stream)


def _split_ctas(pkv, wl, bt, cl):
    """Reference output through the workspace entry, and how many CTAs of
    that launch merged a context split (workspace meta rows with s >= 0)."""
    Hq, Hkv, D = wl.q.shape[-2], wl.k_pool.shape[1], wl.k_pool.shape[3]
    ws = torch.empty(pkv.workspace_size(Hq, Hkv, 1, D), dtype=torch.uint8, device="cuda")
    ref = pkv.paged_decode_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale, workspace=ws)
    torch.cuda.synchronize()
    grid = torch.cuda.get_device_properties(0).multi_processor_count
    meta = ws[:grid * 16].view(torch.int32).view(grid, 4).cpu().numpy()
    return ref, int((meta[:, 0] >= 0).sum())


@pytest.mark.parametrize("name,kw,warm_kw", [
    ("llama70b_gqa", {"B": 24, "max_len": 3000}, {"name": "llama7b_mha", "B": 5, "max_len": 900}),
    ("llama7b_mha", {"B": 8, "max_len": 2000}, {"name": "llama70b_gqa", "B": 40, "max_len": 700}),
    # 8-token blocks: the head-pair form (two KV heads per staged tile, 16 rows)
    ("llama70b_gqa_bs8", {"B": 24, "max_len": 3000}, {"name": "llama7b_mha", "B": 5, "max_len": 900}),
    # MQA at head_dim 128: 32 query rows per KV head, the largest shape the
    # fixed scratch admits; long enough that every CTA splits a context
    ("llama70b_gqa", {"lens": np.full(6, 9000, np.int32), "Hq": 32, "Hkv": 1, "seed": 41},
     {"name": "long_verify", "B": 1, "q_len": 1, "max_len": 20000}),
])
def test_static_scratch_matches_workspace_entry_and_oracle(name, kw, warm_kw):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import paged_kv_cache_371_b200 as pkv
    L = pkv.lib()
    warm_kw = dict(warm_kw)
    warm = make_workload(warm_kw.pop("name"), "cuda", **warm_kw)
    wbt = torch.as_tensor(warm.block_tables, device="cuda")
    wcl = torch.as_tensor(warm.lens, device="cuda")
    wout = torch.empty_like(warm.q)
    assert _call_static(L, warm, wbt, wcl, wout) == 0, L.kv_last_error_string()

    wl = make_workload(name, "cuda", **kw)
    bt = torch.as_tensor(wl.block_tables, device="cuda")
    cl = torch.as_tensor(wl.lens, device="cuda")
    ref, n_split = _split_ctas(pkv, wl, bt, cl)
    assert n_split > 0, "the checked shape must split contexts across CTAs"
    exact = oracle_subset(wl, list(range(wl.B)))
    for call in range(2):
        out = torch.full_like(wl.q, float("nan"))
        rc = _call_static(L, wl, bt, cl, out)
        assert rc == 0, L.kv_last_error_string()
        torch.cuda.synchronize()
        assert pkv.device_error() == 0
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"call {call}: bits differ"
        assert_close(out, exact, f"static scratch, call {call}")


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
