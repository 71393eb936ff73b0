"""Multi-rank host logic of bench.py on CPU: two gloo ranks, each with its own
replica of the workload (weak scaling, no data-path collective); the job
totals are the ranks' sums over the slowest rank's time."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from workloads import make_workload
        from workloads.synth import CONFIGS
        spec = CONFIGS["llama70b_gqa"]
        seed = bench.rank_seed(spec.seed, rank)
        wl = make_workload("llama70b_gqa", "cpu", B=6, max_len=200, seed=seed, Hq=8, Hkv=2, D=64)
        kvb, allb = bench.algorithmic_bytes(wl.lens, 8, 2, 64, wl.spec.bs, 1)
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        kv_all, th_all, t_all = bench.aggregate(kvb, int(wl.lens.sum()) * 8, ms, world, "cpu")
        q.put((rank, seed, wl.lens.tolist(), kvb, kv_all, th_all, t_all))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_replicas():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, q), nprocs=2, join=True, start_method="spawn")
    res = sorted(q.get(timeout=60) for _ in range(2))
    (r0, s0, l0, kb0, kv0, th0, t0), (r1, s1, l1, kb1, kv1, th1, t1) = res
    assert s0 != s1 and l0 != l1                # independent replicas
    assert kv0 == kv1 == kb0 + kb1              # bytes summed over ranks
    assert th0 == th1 == (sum(l0) + sum(l1)) * 8
    assert t0 == t1 == 15.0                     # slowest rank's time


def test_algorithmic_bytes_counts_kv_q_out_tables():
    import bench
    kv, allb = bench.algorithmic_bytes([16, 17], Hq=4, Hkv=2, D=64, bs=16, q_len=1)
    assert kv == (16 + 17) * 2 * 64 * 2 * 2
    assert allb == kv + 2 * 1 * 4 * 64 * 2 * 2 + (1 + 2) * 4 + 2 * 4
