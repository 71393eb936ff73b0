"""Test inputs whose attention scores jump late in the context.

The online softmax ("大模型推理加速与显存黑科技 (Inference Acceleration & KV
Cache)" §4.2) keeps a running maximum and rescales everything accumulated so
far whenever the maximum grows.  With N(0,1) queries and keys the maximum
settles within the first tile, so later rescales (and, in the prefill
kernel, the lazy rescale that only fires when a row's maximum grows by more
than 2^8) are never reached.  These helpers reshape a workload's inputs so
that they are:

* ``plant``: every query row of a (sequence, KV head) gets a common direction
  u (a seeded unit vector): q += b*u.  The key of each chosen token t becomes
  c*u, so its score for every row of that KV head is about scale*c*b, far
  above the other tokens' N(0,1)-sized scores.  Growing gains at later tokens
  make the maximum jump several times along the context.
* ``ramp``: key t of every sequence is multiplied by (1 + t/rate), so the
  scores' spread, and with it the running maximum, grows steadily.

Only inputs change; the oracle and the CUDA path read the same modified
tensors.  No attention arithmetic here.
"""
from __future__ import annotations

import numpy as np
import torch


def plant(wl, plan, b=3.0, seed=0):
    """plan: {sequence: [(token, gain), ...]}.  Modifies wl.q and wl.k_pool
    in place (all KV heads of each planted token)."""
    B, q_len, Hq, D = wl.q.shape
    nb, Hkv, bs, _ = wl.k_pool.shape
    G = Hq // Hkv
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    u = torch.randn((B, Hkv, D), generator=g, dtype=torch.float64)
    u /= u.norm(dim=-1, keepdim=True)
    q = wl.q.double().cpu() + b * u.repeat_interleave(G, dim=1)[:, None, :, :]
    wl.q = q.to(torch.float16).to(wl.q.device)
    for s, items in plan.items():
        for t, c in items:
            t = int(t)
            assert 0 <= t < int(wl.lens[s]), (s, t)
            blk = int(wl.block_tables[s, t // bs])
            wl.k_pool[blk, :, t % bs, :] = (c * u[s]).to(torch.float16).to(wl.k_pool.device)
    return wl


def ramp(wl, rate):
    """Scale key t of every sequence by (1 + t / rate).  Each block must
    belong to one sequence (no shared prefix)."""
    nb, Hkv, bs, D = wl.k_pool.shape
    seen = set()
    for s in range(wl.B):
        n = -(-int(wl.lens[s]) // bs)
        ids = wl.block_tables[s, :n].astype(np.int64)
        assert not (seen & set(ids.tolist())), "ramp needs private blocks"
        seen.update(ids.tolist())
        t = np.arange(n * bs, dtype=np.float64).reshape(n, bs)
        f = torch.as_tensor(1.0 + t / rate, dtype=torch.float32, device=wl.k_pool.device)
        idx = torch.as_tensor(ids, device=wl.k_pool.device)
        k = wl.k_pool[idx].float() * f[:, None, :, None]
        wl.k_pool[idx] = k.to(torch.float16)
    return wl
