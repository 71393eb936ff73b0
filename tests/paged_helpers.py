"""Shared helpers of the GPU parity tests: run the CUDA path, run the oracle
on (a sample of) the same inputs, compare with the stated tolerance."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Attention tolerance: fp16 in, fp32 accumulate, fp16 out, against exact fp64
# attention: |gpu - ref| <= ATOL + RTOL * |ref|.
ATOL = 2e-3
RTOL = 1e-2


def device_inputs(wl, device="cuda"):
    bt = torch.as_tensor(wl.block_tables, device=device)
    cl = torch.as_tensor(wl.lens, device=device)
    return bt, cl


def oracle_subset(wl, seqs, q_len=1, lens=None, tables=None, q=None):
    """Oracle output for the sequences ``seqs`` of a (device) workload: their
    blocks are copied to the host and the tables renumbered (plain data
    movement; every value the oracle reads comes from the generator)."""
    seqs = np.asarray(seqs)
    tables = (wl.block_tables if tables is None else tables)[seqs]
    lens = (wl.lens if lens is None else lens)[seqs]
    ids = np.unique(tables[tables >= 0])
    idx = torch.as_tensor(ids, device=wl.k_pool.device, dtype=torch.long)
    K = wl.k_pool[idx].cpu().numpy()
    V = wl.v_pool[idx].cpu().numpy()
    t2 = np.where(tables >= 0, np.searchsorted(ids, np.maximum(tables, 0)), -1).astype(np.int32)
    qq = (wl.q if q is None else q)[torch.as_tensor(seqs, device=wl.q.device)].cpu().numpy()
    return oracle.paged_attention(qq, K, V, t2, lens.astype(np.int32), scale=wl.scale,
                                  q_len=q_len)


def assert_close(gpu: torch.Tensor, ref: np.ndarray, what=""):
    g = gpu.detach().float().cpu().numpy().astype(np.float64).reshape(ref.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst at {i}: "
                             f"gpu {g[i]!r} ref {ref[i]!r}")
    return float(err.max())
