#!/usr/bin/env python
"""Benchmark of the paged decode hot path on B200.

One step = one decode step of one attention layer over a batch:
  copy-on-write block copies (when the step has any) -> cache append of one
  new token per sequence -> paged decode (or verify) attention over the
  grown contexts (+ the split-context merge).
The device-timed steps replay slots and tables the host block manager
reserved before timing; the e2e figure runs the whole step through the
public API with host buffers, the host reservation (and, for beam search,
the beam reorder) of every step inside its timed region.  The default run
also times the Llama-2-70B-shaped GQA decode at block sizes 16 and 8
(`targets` in the JSON line).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                       [--impl ours|reference]
Multi-GPU (weak scaling, independent replicas, no data-path collective):
  torchrun --nproc-per-node N bench.py --gpus N ...
Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged decode attention KV GB/s and % of B200 HBM peak; tokens·heads/s"
DEFAULT_WORKLOAD = "llama7b_mha"
FALLBACK_HBM_GBS = 6650.0
CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-targets", action="store_true",
                    help="skip the 70B GQA decode lines reported beside the default workload")
    ap.add_argument("--batch", type=int, default=0,
                    help="use only the first B sequences of the workload (profiling runs)")
    ap.add_argument("--consumer", type=int, default=0, choices=[0, 1, 2],
                    help="compute path for several query rows per KV head: 1 warp-level MMAs, "
                         "2 tcgen05 with tensor-memory accumulators, 0 the library's default")
    return ap.parse_args(argv)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank runs its own replica of the workload (weak scaling)."""
    return base_seed + 7919 * rank


def algorithmic_bytes(lens, Hq, Hkv, D, bs, q_len, k_bytes=2):
    """(K/V bytes read, all bytes) of one attention launch: K and V rows of
    every visible token, q and out, the used table entries and the lengths
    (k_bytes = 1: int8 K codes, plus the fp32 channel scales)."""
    L = [int(x) for x in lens]
    kv = sum(L) * Hkv * D * (k_bytes + 2)
    qo = len(L) * q_len * Hq * D * 2 * 2
    tab = sum(-(-x // bs) for x in L) * 4 + len(L) * 4
    scales = Hkv * D * 4 if k_bytes == 1 else 0
    return kv, kv + qo + tab + scales


def split_workload(name):
    """'<config>' or '<config>_q8k' (the same config with an int8 K pool)."""
    return (name[:-4], True) if name.endswith("_q8k") else (name, False)


def pool_tokens(pool):
    """[num_blocks][Hkv][bs][D] -> [num_blocks*bs][Hkv][D] in slot order (a copy)."""
    nb, Hkv, bs, D = pool.shape
    return pool.permute(0, 2, 1, 3).reshape(nb * bs, Hkv, D).contiguous()


def quantise_pool_device(pkv, wl):
    """int8 K pool of the workload through the library: channel scales from
    every pool token, then the quantising append of every slot."""
    import torch
    nb, Hkv, bs, D = wl.k_pool.shape
    kt, vt = pool_tokens(wl.k_pool), pool_tokens(wl.v_pool)
    sc = pkv.paged_kv_k_scales(kt)
    kq = torch.empty((nb, Hkv, bs, D), dtype=torch.int8, device=wl.k_pool.device)
    slots = torch.arange(nb * bs, dtype=torch.int64, device=wl.k_pool.device)
    pkv.paged_kv_append_q8k(kt, vt, slots, sc, kq, wl.v_pool)
    del kt, vt
    return kq, sc


def quantise_pool_host(K):
    """The same with the oracle on host arrays: (codes, scales)."""
    import numpy as np
    import oracle
    n, Hkv, bs, D = K.shape
    toks = K.transpose(0, 2, 1, 3).reshape(n * bs, Hkv, D).copy()
    sc = oracle.k_scales(toks)
    K8, _ = oracle.append_q8k(np.zeros(K.shape, np.int8), np.zeros_like(K), toks, toks,
                              np.arange(n * bs, dtype=np.int64), sc)
    return K8, sc


def prefill_flops(lens, Hq, D, q_len):
    """Flops of causal chunked prefill: every row j of a sequence of length L
    sees L - q_len + j + 1 tokens; q.K and P.V cost 2*D flops per token each."""
    tot = 0
    for L in lens:
        L = int(L)
        seen = q_len * (L - q_len) + q_len * (q_len + 1) // 2
        tot += seen * Hq * D * 4
    return tot


def measured_tensor_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (cuBLAS bf16 burst; fp16 runs at the same dense rate)"
    except Exception:
        return 1590.0, "fallback"


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_sha(kernel="paged_attention.cu"):
    h = hashlib.sha256()
    for name in (kernel, "kv_ptx.cuh"):
        with open(os.path.join(ROOT, "paged_kv_cache_371_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload, kernel="paged_attention.cu"):
    """DRAM bytes per launch of the attention kernel from a committed ncu
    summary, if it was taken on the current kernel source (else None)."""
    sha = kernel_source_sha(kernel)
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        kv = {}
        with open(path, encoding="utf-8") as f:
            for line in f:
                if ":" in line and line.startswith("- "):
                    k, v = line[2:].split(":", 1)
                    kv[k.strip()] = v.strip().strip("`")
        if (kv.get("workload") == workload and kv.get("kernel_source_sha256") == sha
                and "traffic_bytes_per_launch" in kv):
            try:
                return int(float(kv["traffic_bytes_per_launch"]))
            except ValueError:
                return None
    return None


class ClockSampler:
    """Samples SM clock, max clock and throttle reasons every ~1 ms through
    NVML while the timed region runs (nvidia-smi's 200 ms period is longer
    than a short timed region)."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index):
        self.dev = device_index
        self.samples = []
        self.max_mhz = None
        self._stop = None

    def _handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            idx = int(vis.split(",")[self.dev]) if vis else self.dev
            return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def _run(self, h):
        import pynvml
        while not self._stop.is_set():
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, rs))
            except Exception:
                pass
            time.sleep(0.001)

    def __enter__(self):
        import threading
        try:
            import pynvml
            h = self._handle()
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._stop = threading.Event()
            self._t = threading.Thread(target=self._run, args=(h,), daemon=True)
            self._t.start()
        except Exception:
            self._stop = None
        return self

    def __exit__(self, *exc):
        if self._stop is not None:
            self._stop.set()
            self._t.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "source": "nvml"}
        reasons = sorted(n for n, bit in self.REASONS.items()
                         if any(r & bit for _, r in self.samples))
        return {"sm_mhz": statistics.median(sm for sm, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples),
                "source": "nvml, 1 ms polling during the timed steps"}


def aggregate(kv_bytes, tokens_heads, total_ms, world, device):
    """Whole-job totals: bytes and tokens of all ranks, time of the slowest
    rank (each rank times its own replica on the device).  Host-side only;
    no data-path collective."""
    import torch
    import torch.distributed as dist
    tot = torch.tensor([float(kv_bytes), float(tokens_heads)], dtype=torch.float64, device=device)
    tmax = torch.tensor([float(total_ms)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(tot, op=dist.ReduceOp.SUM)
        dist.all_reduce(tmax, op=dist.ReduceOp.MAX)
    kv_all, th_all = tot.tolist()
    return kv_all, th_all, tmax.item()


# ---------------------------------------------------------------------------
# our arm

def adopt_workload(pkv, wl, extra_cap):
    """Host block manager in the state the generator's placement describes:
    the same ids, allocated in the same order (prefix blocks forked)."""
    import numpy as np
    bs = wl.spec.bs
    B = wl.B
    cap = wl.block_tables.shape[1] + extra_cap
    pool = pkv.KVPool(wl.num_blocks, bs, num_kv_heads=wl.spec.Hkv, head_dim=wl.q.shape[-1],
                      order=wl.order)
    tables = np.full((B, cap), -1, np.int32)
    nblk = np.zeros(B, np.int32)
    P = wl.extra.get("prefix_blocks", 0)
    prefix = pool.alloc(P) if P else []
    for s in range(B):
        need = int(-(-int(wl.lens[s]) // bs))
        if P:
            if s:
                pool.fork(prefix)
            tables[s, :P] = prefix
        ids = pool.alloc(need - P)
        tables[s, P:need] = ids
        nblk[s] = need
        assert tables[s, :need].tolist() == wl.block_tables[s, :need].tolist()
    return pool, tables, nblk


BEAMS = 8  # beams per prompt of the beam_search config


def build_beam_steps(pkv, wl, n_steps, device, seed, width=BEAMS):
    """Per-step inputs of beam search over the workload's prompts: each step
    the survivors are drawn (seeded) within each prompt's beams, the host
    block manager reorders the tables (kv_beam_reorder) and reserves one slot
    per beam (copy-on-write pairs for shared partial last blocks)."""
    import numpy as np
    import torch
    from workloads import normal_fp16
    Hq, Hkv, D = wl.q.shape[-2], wl.spec.Hkv, wl.q.shape[-1]
    pool, tables, nblk = adopt_workload(pkv, wl, extra_cap=n_steps // wl.spec.bs + 3)
    S = wl.B
    all_parents = beam_parents(S, width, n_steps, seed)
    beam_len = wl.lens.astype(np.int32)
    steps = []
    for i in range(n_steps):
        parents = all_parents[i]
        tables, nblk = pool.beam_reorder(tables, nblk, parents)
        lens = beam_len[parents].astype(np.int32)
        slots, pairs = pool.reserve_slots(tables, nblk, lens)
        beam_len = lens + 1
        n = S * width
        steps.append({
            "q": normal_fp16((n, 1, Hq, D), seed * 100003 + 3 * i, device),
            "k_new": normal_fp16((n, Hkv, D), seed * 100003 + 3 * i + 1, device),
            "v_new": normal_fp16((n, Hkv, D), seed * 100003 + 3 * i + 2, device),
            "slots": torch.as_tensor(slots, device=device),
            "pairs": torch.as_tensor(pairs, device=device) if len(pairs) else None,
            "tables": torch.as_tensor(tables.copy(), device=device),
            "lens": torch.as_tensor(beam_len.copy(), device=device),
            "lens_host": beam_len.copy(),
            "tables_host": tables.copy(),
        })
    return steps


def build_steps(pkv, wl, n_steps, device, seed):
    """Per-step inputs: slots / copy pairs from the host block manager, new
    K/V, queries, tables and lengths after the append."""
    import numpy as np
    import torch
    from workloads import normal_fp16
    bs = wl.spec.bs
    Hq, Hkv, D = wl.q.shape[-2], wl.spec.Hkv, wl.q.shape[-1]
    q_len = wl.q.shape[1]
    pool, tables, nblk = adopt_workload(pkv, wl, extra_cap=n_steps // bs + 2)
    lens = wl.lens.astype(np.int32).copy()
    steps = []
    for i in range(n_steps):
        slots, pairs = pool.reserve_slots(tables, nblk, lens)
        lens = lens + 1
        st = {
            "q": normal_fp16((wl.B, q_len, Hq, D), seed * 100003 + 3 * i, device),
            "k_new": normal_fp16((wl.B, Hkv, D), seed * 100003 + 3 * i + 1, device),
            "v_new": normal_fp16((wl.B, Hkv, D), seed * 100003 + 3 * i + 2, device),
            "slots": torch.as_tensor(slots, device=device),
            "pairs": torch.as_tensor(pairs, device=device) if len(pairs) else None,
            "tables": torch.as_tensor(tables.copy(), device=device),
            "lens": torch.as_tensor(lens.copy(), device=device),
            "lens_host": lens.copy(),
            "tables_host": tables.copy(),
        }
        steps.append(st)
    return steps


def run_prefill(args):
    """Chunked prefill: append the chunk's K/V, then causal attention of the
    chunk over the paged cache; reported in TFLOP/s against the tensor peak."""
    import numpy as np
    import torch
    import paged_kv_cache_371_b200 as pkv
    from workloads import make_workload, normal_fp16
    from workloads.synth import CONFIGS
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    spec = CONFIGS[args.workload]
    wl = make_workload(args.workload, device, seed=rank_seed(spec.seed, rank), B=args.batch or None)
    q_len, Hq, Hkv, D, bs = spec.q_len, spec.Hq, spec.Hkv, spec.D, spec.bs
    bt, cl = torch.as_tensor(wl.block_tables, device=device), torch.as_tensor(wl.lens, device=device)
    # slots of the chunk's tokens (positions L - q_len .. L - 1 of each sequence)
    slots = []
    for s_, L in enumerate(wl.lens):
        for t in range(int(L) - q_len, int(L)):
            slots.append(int(wl.block_tables[s_, t // bs]) * bs + t % bs)
    slots = torch.as_tensor(np.array(slots, np.int64), device=device)
    kn = normal_fp16((len(slots), Hkv, D), 901, device)
    vn = normal_fp16((len(slots), Hkv, D), 902, device)
    out = torch.empty_like(wl.q)
    flush = L2Flush(device)
    stream = torch.cuda.current_stream(device)

    def step(ev=None):
        pkv.paged_kv_append(kn, vn, slots, wl.k_pool, wl.v_pool)
        if ev is not None:
            ev.record(stream)
        pkv.paged_prefill_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale, q_len, out=out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert pkv.device_error() == 0
    es = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ea = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ee = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with ClockSampler(local) as clk:
        for k in range(args.steps):
            flush()
            es[k].record(stream)
            step(ea[k])
            ee[k].record(stream)
        torch.cuda.synchronize()
    assert pkv.device_error() == 0
    step_ms = [es[k].elapsed_time(ee[k]) for k in range(args.steps)]
    attn_ms = [ea[k].elapsed_time(ee[k]) for k in range(args.steps)]
    fl = prefill_flops(wl.lens, Hq, D, q_len)
    peak, kind = measured_tensor_peak()
    tot_fl, _, t_all = aggregate(fl * args.steps, 0, sum(step_ms), world, device)
    value = tot_fl / (t_all * 1e-3) / 1e12
    achieved = fl / (statistics.mean(attn_ms) * 1e-3) / 1e12

    # e2e: the chunk's queries and K/V from pinned host memory, the output back
    e2e = None
    if not args.no_e2e:
        hq, hk, hv, hs = (x.cpu().pin_memory() for x in (wl.q, kn, vn, slots))
        dq, dk, dv, ds = (torch.empty_like(x) for x in (wl.q, kn, vn, slots))
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hs))
        times = []
        for k in range(args.warmup + args.steps):
            flush()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for d_, h_ in ((dq, hq), (dk, hk), (dv, hv), (ds, hs)):
                d_.copy_(h_, non_blocking=True)
            pkv.paged_kv_append(dk, dv, ds, wl.k_pool, wl.v_pool)
            pkv.paged_prefill_attention(dq, wl.k_pool, wl.v_pool, bt, cl, wl.scale, q_len, out=out)
            hout.copy_(out, non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize()
            if k >= args.warmup:
                times.append(e0.elapsed_time(e1))
        e_fl, _, e_t = aggregate(fl * args.steps, 0, sum(times), world, device)
        e2e = {"value": round(e_fl / (e_t * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": hout.numel() * hout.element_size()}
    if rank != 0:
        return None
    res = {
        "metric": "paged prefill attention TFLOP/s", "value": round(value, 2), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t_all / args.steps, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": args.workload, "description": spec.description, "B": wl.B,
                   "Hq": Hq, "Hkv": Hkv, "head_dim": D, "block_size": bs, "q_len": q_len,
                   "mean_context": float(np.mean(wl.lens)),
                   "step": "append the chunk's K/V + causal paged prefill attention",
                   "l2": f"flushed before every timed step by reading {flush.bytes >> 20} MiB "
                         "(a sum into one word: no dirty lines left)"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": ncu_traffic(args.workload, "paged_prefill.cu"),
                     "kernel": "paged_prefill_kernel (tcgen05)", "peak_kind": kind},
        "gpu_launches": 2 * args.steps,
        "clocks": clk.summary(),
    }
    if e2e:
        res["e2e"] = e2e
    if world == 1 and args.cpu_seconds > 0:
        res["cpu_baseline"] = prefill_cpu_baseline(wl, q_len, args.cpu_seconds)
    return res


def prefill_window(wl, q_len, n_seq, n_pos):
    """Host inputs of a bounded prefill sample: the first n_pos positions of
    the chunks of the first n_seq sequences (their rows see exactly what they
    see in the full chunk: lengths cut to L - q_len + n_pos)."""
    import numpy as np
    import torch
    seqs = np.arange(n_seq)
    tables = wl.block_tables[seqs]
    lens = (wl.lens[seqs] - q_len + n_pos).astype(np.int32)
    ids = np.unique(tables[tables >= 0])
    idx = torch.as_tensor(ids, device=wl.k_pool.device, dtype=torch.long)
    K = wl.k_pool[idx].cpu().numpy()
    V = wl.v_pool[idx].cpu().numpy()
    t2 = np.where(tables >= 0, np.searchsorted(ids, np.maximum(tables, 0)), -1).astype(np.int32)
    q = wl.q[:n_seq, :n_pos].cpu().numpy().copy()
    return q, K, V, t2, lens


def prefill_cpu_baseline(wl, q_len, target_s):
    """The oracle over a bounded sample of this run's chunked prefill,
    repeated to about target_s seconds; reported in TFLOP/s."""
    import oracle
    Hq, D = wl.q.shape[-2], wl.q.shape[-1]
    n_pos = 16
    q, K, V, t2, lens = prefill_window(wl, q_len, 1, n_pos)
    reps, spent = 0, 0.0
    while reps == 0 or spent < target_s:
        t0 = time.perf_counter()
        oracle.paged_attention(q, K, V, t2, lens, scale=wl.scale, q_len=n_pos)
        spent += time.perf_counter() - t0
        reps += 1
    fl = prefill_flops(lens, Hq, D, n_pos) * reps
    return {"value": round(fl / spent / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle", "cpu_model": cpu_model(),
            "sample": f"the first {n_pos} positions of sequence 0's chunk (all {Hq} heads, "
                      f"{int(lens[0])} tokens) x {reps} repeat(s), fp64 C oracle, {spent:.2f} s"}


def beam_parents(S, width, n_steps, seed):
    """The beams each step continues: step 0 forks every prompt into `width`
    beams; later steps draw the survivors (seeded) within each prompt's beams
    (the sampler's decision, made by the caller, not by the library)."""
    import numpy as np
    rng = np.random.Generator(np.random.PCG64(seed + 7))
    out = [np.repeat(np.arange(S), width).astype(np.int32)]
    for _ in range(n_steps - 1):
        out.append(np.concatenate([g * width + rng.integers(0, width, size=width)
                                   for g in range(S)]).astype(np.int32))
    return out


class L2Flush:
    """Evicts L2 between timed steps by READING a buffer of twice its size
    into a one-word sum: no dirty lines are left behind for the next timed
    step to write back."""

    def __init__(self, device):
        import torch
        l2 = torch.cuda.get_device_properties(device).L2_cache_size
        n = max(2 * l2, 256 << 20) // 4
        self.buf = torch.zeros(n, dtype=torch.float32, device=device)
        self.acc = torch.zeros((), dtype=torch.float32, device=device)
        self.bytes = n * 4

    def __call__(self):
        import torch
        torch.sum(self.buf, 0, out=self.acc)


def unique_kv_bytes(tables, lens, bs, Hkv, D, k_bytes=2):
    """K/V bytes of the distinct cache rows one launch reads: a block shared
    by several sequences (a common prefix, beams) counts once, with the most
    rows any of them reads from it."""
    import numpy as np
    rows = {}
    for s in range(len(lens)):
        L = int(lens[s])
        n = -(-L // bs)
        for b in range(n):
            blk = int(tables[s, b])
            used = min(bs, L - b * bs)
            if rows.get(blk, 0) < used:
                rows[blk] = used
    return sum(rows.values()) * Hkv * D * (k_bytes + 2)


TARGET_WORKLOADS = ("llama70b_gqa", "llama70b_gqa_bs8")


def run_ours(args):
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    try:
        result = measure_decode(args, args.workload, rank, world, local, device, full=True)
        if args.workload == DEFAULT_WORKLOAD and not args.no_targets and not args.batch:
            # the Llama-2-70B-shaped GQA decode at both block sizes, same
            # steps and warm-up, reported beside the headline
            targets = {}
            for name in TARGET_WORKLOADS:
                torch.cuda.empty_cache()
                r = measure_decode(args, name, rank, world, local, device, full=False)
                if rank == 0:
                    targets[name] = {k: r[k] for k in ("value", "unit", "ms_per_step", "hbm_frac",
                                                       "tokens_heads_per_s", "roofline", "clocks",
                                                       "gpu_launches", "config")}
            if rank == 0:
                result["targets"] = targets
    finally:
        if world > 1:
            dist.destroy_process_group()
    return result if rank == 0 else None


def measure_decode(args, workload, rank, world, local, device, full=True):
    """Device-timed decode steps of one workload (+ with `full`: the
    end-to-end serving loop and, on one GPU, the oracle baseline)."""
    import numpy as np
    import torch
    import torch.distributed as dist

    import paged_kv_cache_371_b200 as pkv
    from workloads import make_workload
    from workloads.synth import CONFIGS

    base, q8k = split_workload(workload)
    spec = CONFIGS[base]
    seed = rank_seed(spec.seed, rank)
    beams = base == "beam_search"
    n_distinct = min(args.warmup + args.steps, 64)
    do_e2e = full and not args.no_e2e
    n_host = args.warmup + args.steps if do_e2e else n_distinct  # steps the host pool must fit
    B = args.batch or spec.B
    if beams:
        spare = (n_host // spec.bs + 3) * BEAMS * B * 2
    else:
        spare = (n_host // spec.bs + 2) * B
    wl = make_workload(base, device, seed=seed, B=args.batch or None, spare_blocks=spare)
    q_len = spec.q_len
    Hq, Hkv, D, bs = spec.Hq, spec.Hkv, spec.D, spec.bs
    k_bytes = 1 if q8k else 2
    steps = (build_beam_steps(pkv, wl, n_distinct, device, seed) if beams
             else build_steps(pkv, wl, n_distinct, device, seed))
    kq = ksc = None
    if q8k:
        kq, ksc = quantise_pool_device(pkv, wl)
    n_rows = steps[0]["q"].shape[0]  # sequences (beams) attended per step
    out = torch.empty((n_rows, q_len, Hq, D), dtype=torch.float16, device=device)
    ws = torch.empty(pkv.workspace_size(Hq, Hkv, q_len, D), dtype=torch.uint8, device=device)
    flush = L2Flush(device)
    stream = torch.cuda.current_stream(device)

    def step(i, ev=None):
        st = steps[i % n_distinct]
        decode_step(pkv, wl, st["q"], st["k_new"], st["v_new"], st["slots"], st["tables"],
                    st["lens"], st["pairs"], out, ws, q_len, kq, ksc, ev, stream)

    for i in range(args.warmup):
        flush()
        step(i)
    torch.cuda.synchronize()
    assert pkv.device_error() == 0, "device error during warm-up"

    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    launches = 0
    n_cow = 0
    kv_bytes_total = 0
    alg_attn = []
    th_tokens = 0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for k in range(args.steps):
            i = args.warmup + k
            st = steps[i % n_distinct]
            flush()
            ev_s[k].record(stream)
            step(i)
            ev_e[k].record(stream)
            launches += 3 + (1 if st["pairs"] is not None else 0)
            n_cow += 0 if st["pairs"] is None else int(st["pairs"].shape[0])
            kvb, allb = algorithmic_bytes(st["lens_host"], Hq, Hkv, D, bs, q_len, k_bytes)
            kv_bytes_total += kvb
            alg_attn.append(allb)
            th_tokens += int(st["lens_host"].sum()) * Hq * q_len
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        # the attention launch (+ its split merge) alone, for the roofline:
        # the same inputs, L2 flushed before each (inside a step it overlaps
        # its set-up with the append's tail, which an event between the two
        # would both split and serialise)
        ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ev_b = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        for k in range(args.steps):
            st = steps[(args.warmup + k) % n_distinct]
            flush()
            ev_a[k].record(stream)
            attention_call(pkv, wl, st["q"], st["tables"], st["lens"], out, ws, q_len, kq, ksc)
            ev_b[k].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    step_ms = [ev_s[k].elapsed_time(ev_e[k]) for k in range(args.steps)]
    attn_ms = [ev_a[k].elapsed_time(ev_b[k]) for k in range(args.steps)]
    err = pkv.device_error()
    assert err == 0, f"device error word {err}"
    total_ms = sum(step_ms)

    kv_all, th_all, t_all = aggregate(kv_bytes_total, th_tokens, total_ms, world, device)
    value = kv_all / (t_all * 1e-3) / 1e9

    e2e = None
    if do_e2e:
        e2e = run_e2e(pkv, wl, steps, n_distinct, args, ws, stream, device, Hq, Hkv, D, bs, q_len,
                      world, kq, ksc, beams, seed)

    peak, peak_kind = measured_hbm_peak()
    attn_avg_ms = statistics.mean(attn_ms)
    achieved = statistics.mean(alg_attn) / (attn_avg_ms * 1e-3) / 1e9
    result = None
    if rank == 0:
        st_last = steps[-1]
        tables_last = st_last["tables_host"]
        shared = base in ("prefix_beam", "beam_search")
        result = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(t_all / args.steps, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": {
                "workload": workload + (f"[B={wl.B}]" if args.batch else ""),
                "description": spec.description, "B": n_rows,
                "Hq": Hq, "Hkv": Hkv, "head_dim": D, "block_size": bs, "q_len": q_len,
                "mean_context": float(np.mean(st_last["lens_host"])),
                "cow_copies_per_step": round(n_cow / args.steps, 2),
                "step": "copy-on-write copies + append 1 token/sequence + paged attention + merge",
                "k_pool": ("int8 codes, fp32 scale per (KV head, channel); V fp16" if q8k
                           else "fp16"),
                "l2": f"flushed before every timed step by reading {flush.bytes >> 20} MiB "
                      "(a sum into one word: no dirty lines left)",
                "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                "consumer": consumer_path(Hq // Hkv * q_len, D, q8k)},
            "hbm_frac": round(value / peak, 4),
            "hbm_peak_gbs": peak, "hbm_peak_kind": peak_kind,
            "tokens_heads_per_s": round(th_all / (t_all * 1e-3), 1),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                         "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "traffic": ncu_traffic(workload),
                         "kernel": "paged_attention_kernel + lse_merge_kernel",
                         "attention_ms": round(attn_avg_ms, 5),
                         "timing": "the attention launch and its merge alone, a loop of `steps` "
                                   "launches after the step loop, L2 flushed before each",
                         "peak_kind": peak_kind},
            "gpu_launches": launches,
            "clocks": clk.summary(),
        }
        if shared:
            # the same launch counted in distinct cache rows (shared blocks once)
            ub = unique_kv_bytes(tables_last, st_last["lens_host"], bs, Hkv, D, k_bytes)
            lb = algorithmic_bytes(st_last["lens_host"], Hq, Hkv, D, bs, q_len, k_bytes)[0]
            u_gbs = ub / (attn_avg_ms * 1e-3) / 1e9
            result["roofline"]["unique_kv_bytes"] = ub
            result["roofline"]["logical_kv_bytes"] = lb
            result["roofline"]["unique_gbs"] = round(u_gbs, 2)
            result["roofline"]["unique_frac"] = round(u_gbs / peak, 4)
        if e2e:
            result["e2e"] = e2e
        if full and world == 1 and args.cpu_seconds > 0:
            # the timed appends only wrote slots past each sequence's original
            # length, so the workload's original tokens are still in the pools
            if beams:  # the oracle over the beams of the last step
                wl.block_tables = steps[-1]["tables_host"]
                wl.lens = steps[-1]["lens_host"]
                wl.q = steps[-1]["q"]
            result["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds, q8k)
    del steps, wl, kq, ksc, out, ws, flush
    return result


CONSUMER = 0  # --consumer (0: the library's default path)


def consumer_path(rows, D, q8k):
    """Which compute path the attention launch takes (mirrors the library's
    default choice: the warp-level MMAs unless --consumer 2)."""
    if rows == 1:
        return "fma (one query row per KV head)"
    if D != 128:
        return "mma.sync"
    c = CONSUMER or 1
    return "tcgen05 (tensor memory)" if c == 2 else "mma.sync"


def decode_step(pkv, wl, q, k_new, v_new, slots, tables, lens, pairs, out, ws, q_len, kq, ksc,
                ev=None, stream=None):
    """One decode step through the public API: copy-on-write copies, append
    of the new tokens, attention (int8 K pool when kq is given)."""
    if kq is None:
        if pairs is not None:
            pkv.paged_kv_copy_blocks(wl.k_pool, wl.v_pool, pairs)
        pkv.paged_kv_append(k_new, v_new, slots, wl.k_pool, wl.v_pool)
    else:
        if pairs is not None:
            pkv.paged_kv_copy_blocks_q8k(kq, wl.v_pool, pairs)
        pkv.paged_kv_append_q8k(k_new, v_new, slots, ksc, kq, wl.v_pool)
    if ev is not None:
        ev.record(stream)
    attention_call(pkv, wl, q, tables, lens, out, ws, q_len, kq, ksc)


def attention_call(pkv, wl, q, tables, lens, out, ws, q_len, kq, ksc):
    """The attention launch of a decode step (+ its split merge)."""
    if kq is not None:
        pkv.paged_attention_q8k(q, kq, ksc, wl.v_pool, tables, lens, wl.scale, q_len, out=out,
                                workspace=ws, consumer=CONSUMER)
    elif CONSUMER:
        pkv.paged_attention(q, wl.k_pool, wl.v_pool, tables, lens, wl.scale, q_len, out=out,
                            workspace=ws, consumer=CONSUMER)
    elif q_len == 1:
        pkv.paged_decode_attention(q, wl.k_pool, wl.v_pool, tables, lens, wl.scale, out=out,
                                   workspace=ws)
    else:
        pkv.paged_verify_attention(q, wl.k_pool, wl.v_pool, tables, lens, wl.scale, q_len, out=out,
                                   workspace=ws)


def run_e2e(pkv, wl, steps, n_distinct, args, ws, stream, device, Hq, Hkv, D, bs, q_len, world,
            kq=None, ksc=None, beams=False, seed=0):
    """The whole decode step through the public API with host buffers, run
    the way a serving loop runs it.  Every step, inside the timed region:
    the host block manager reserves one slot per sequence (for beam search,
    after reordering the beams' tables), emitting copy-on-write pairs; the
    slots, pairs, tables, lengths and the step's q / K / V go host -> device
    from pinned memory; copy-on-write copies, append, attention and merge run;
    the output comes back device -> host.  Step k+1's host work and input
    copies overlap step k's kernels (double-buffered inputs and outputs, two
    side streams).  The host pool starts from the workload's placement, so
    the first steps reserve the slots the device-timed steps used.  No L2
    flush: each step reads far more K/V than the 126 MB L2."""
    import numpy as np
    import torch
    import torch.distributed as dist
    n_total = args.warmup + args.steps
    pool, tables, nblk = adopt_workload(pkv, wl, extra_cap=n_total // bs + 3)
    lens = wl.lens.astype(np.int32).copy()
    parents = beam_parents(wl.B, BEAMS, n_total, seed) if beams else None
    n = steps[0]["q"].shape[0]
    cap = tables.shape[1]
    # Each step's inputs travel in two copies: q / K / V (the model's outputs
    # of the step, in one pinned block per distinct step) and the bookkeeping
    # (slots, tables, lengths, then the copy-on-write pairs) in one pinned
    # staging block per buffer; each tensor is a 256-byte-aligned view.
    def layout(specs):
        offs, o = {}, 0
        for name, shape, dt in specs:
            nbytes = int(np.prod(shape)) * torch.empty((), dtype=dt).element_size()
            offs[name] = (o, shape, dt, nbytes)
            o += (nbytes + 255) // 256 * 256
        return offs, o

    def views(buf, offs):
        return {k: buf[o:o + nb].view(dt).view(shape) for k, (o, shape, dt, nb) in offs.items()}

    qkv_offs, qkv_bytes = layout([(k, tuple(steps[0][k].shape), steps[0][k].dtype)
                                  for k in ("q", "k_new", "v_new")])
    meta_offs, meta_bytes = layout([("slots", (n,), torch.int64), ("tables", (n, cap), torch.int32),
                                    ("lens", (n,), torch.int32), ("pairs", (n, 2), torch.int32)])
    pairs_off = meta_offs["pairs"][0]
    host_qkv = []
    for st in steps:
        hb = torch.empty(qkv_bytes, dtype=torch.uint8).pin_memory()
        for k, v in views(hb, qkv_offs).items():
            v.copy_(st[k].cpu())
        host_qkv.append(hb)
    stage_buf = [torch.empty(meta_bytes, dtype=torch.uint8).pin_memory() for _ in range(2)]
    stage = [views(b, meta_offs) for b in stage_buf]
    dqkv = [torch.empty(qkv_bytes, dtype=torch.uint8, device=device) for _ in range(2)]
    dmeta = [torch.empty(meta_bytes, dtype=torch.uint8, device=device) for _ in range(2)]
    dbuf = [dict(views(dqkv[b], qkv_offs), **views(dmeta[b], meta_offs)) for b in range(2)]
    data_bytes = sum(nb for (_, _, _, nb) in qkv_offs.values()) + sum(
        meta_offs[k][3] for k in ("slots", "tables", "lens"))
    out0 = torch.empty((n, q_len, Hq, D), dtype=torch.float16, device=device)
    outs = [out0, torch.empty_like(out0)]
    houts = [torch.empty(out0.shape, dtype=out0.dtype).pin_memory() for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_read = [torch.cuda.Event() for _ in range(2)]
    state = {"tables": tables, "nblk": nblk, "lens": lens, "beam_len": lens.copy()}

    def host_step(k, b):
        """Host bookkeeping of step k into staging buffer b; returns (pairs,
        bytes copied host -> device this step)."""
        if beams:
            state["tables"], state["nblk"] = pool.beam_reorder(state["tables"], state["nblk"],
                                                               parents[k])
            cur = state["beam_len"][parents[k]].astype(np.int32)
        else:
            cur = state["lens"]
        slots, pairs = pool.reserve_slots(state["tables"], state["nblk"], cur)
        cur = cur + 1
        if beams:
            state["beam_len"] = cur
        else:
            state["lens"] = cur
        if k >= 2:
            ev_in[b].synchronize()  # step k-2's copies out of staging b are done
        sg = stage[b]
        sg["slots"].numpy()[:] = slots
        sg["tables"].numpy()[:] = state["tables"]
        sg["lens"].numpy()[:] = cur
        npairs = len(pairs)
        if npairs:
            sg["pairs"].numpy()[:npairs] = pairs
        return npairs

    def run(k0, cnt):
        nbytes = 0
        for k in range(k0, k0 + cnt):
            b = k % 2
            npairs = host_step(k, b)
            d = dbuf[b]
            if k - k0 >= 2:
                s_in.wait_event(ev_done[b])      # step k-2 finished reading buffer b
            with torch.cuda.stream(s_in):
                dqkv[b].copy_(host_qkv[k % n_distinct], non_blocking=True)
                mlen = pairs_off + npairs * 8 if npairs else pairs_off
                dmeta[b][:mlen].copy_(stage_buf[b][:mlen], non_blocking=True)
                nbytes = data_bytes + npairs * 8
                pairs = d["pairs"][:npairs] if npairs else None
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if k - k0 >= 2:
                stream.wait_event(ev_read[b])    # step k-2's output was copied out
            if graphs[b] is not None:
                if pairs is not None:            # this step's copy-on-write copies, live
                    if kq is None:
                        pkv.paged_kv_copy_blocks(wl.k_pool, wl.v_pool, pairs)
                    else:
                        pkv.paged_kv_copy_blocks_q8k(kq, wl.v_pool, pairs)
                graphs[b].replay()               # append + attention + merge of buffer b
            else:
                decode_step(pkv, wl, d["q"], d["k_new"], d["v_new"], d["slots"], d["tables"],
                            d["lens"], pairs, outs[b], ws, q_len, kq, ksc)
            ev_done[b].record(stream)
            s_out.wait_event(ev_done[b])
            with torch.cuda.stream(s_out):
                houts[b].copy_(outs[b], non_blocking=True)
                ev_read[b].record(s_out)
        return nbytes

    # The device part of a step on buffer b (append, attention, merge: the
    # same public calls on fixed device buffers) is captured once as a CUDA
    # graph and replayed every step, so the host's per-step work is the
    # bookkeeping, two copies and one graph launch.
    graphs = [None, None]
    graph_note = "eager launches (graph capture failed)"
    try:
        torch.cuda.synchronize()
        for b in range(2):
            d = dbuf[b]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                decode_step(pkv, wl, d["q"], d["k_new"], d["v_new"], d["slots"], d["tables"],
                            d["lens"], None, outs[b], ws, q_len, kq, ksc)
            graphs[b] = g
        graph_note = ("append + attention + merge of each input buffer captured once as a CUDA "
                      "graph and replayed every step; copy-on-write copies launched live before it")
    except Exception as exc:  # the same calls, launched one by one
        graphs = [None, None]
        graph_note = f"eager launches (graph capture failed: {type(exc).__name__})"
        torch.cuda.synchronize()
    run(0, args.warmup)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    lens_at_start = (state["beam_len"] if beams else state["lens"]).copy()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    h2d = run(args.warmup, args.steps)
    s_out.wait_stream(stream)
    e1.record(s_out)
    torch.cuda.synchronize()
    assert pkv.device_error() == 0, "device error in the end-to-end loop"
    # K/V bytes attended: every sequence grows by one token per step
    L0 = lens_at_start.astype(np.int64)
    kvb_total = sum(algorithmic_bytes(L0 + 1 + k, Hq, Hkv, D, bs, q_len, 1 if kq is not None else 2)[0]
                    for k in range(args.steps))
    t = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=device)
    kv = torch.tensor([float(kvb_total)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(kv, op=dist.ReduceOp.SUM)
    pool.close()
    return {"value": round(kv.item() / (t.item() * 1e-3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(out0.numel() * 2),
            "ms_per_step": round(t.item() / args.steps, 5),
            "host_work": ("kv_beam_reorder + " if beams else "") +
                         "kv_batch_reserve_slots every step, inside the timed region",
            "pipelining": "host bookkeeping and input copies of step k+1, and the output copy of "
                          "step k, overlap step k's kernels (double buffers, two side streams); "
                          "L2 not flushed (K/V per step >> L2)",
            "launch": graph_note}


# ---------------------------------------------------------------------------
# oracle timing (CPU baseline and the reference arm)

def oracle_sample(workload, target_s, seed_offset=0):
    """A bounded sample of the workload (fewer sequences, same recipe) sized so
    one oracle call takes about target_s seconds on this host."""
    import oracle
    from workloads import make_workload
    from workloads.synth import CONFIGS
    workload, _ = split_workload(workload)
    spec = CONFIGS[workload]
    probe = make_workload(workload, "cpu", B=1, seed=spec.seed + seed_offset)
    t0 = time.perf_counter()
    oracle.paged_attention(probe.q.numpy(), probe.k_pool.numpy(), probe.v_pool.numpy(),
                           probe.block_tables, probe.lens, scale=probe.scale, q_len=spec.q_len)
    t1 = max(time.perf_counter() - t0, 1e-4)
    n = int(max(1, min(max(1, spec.B // 4), round(target_s / t1))))
    return make_workload(workload, "cpu", B=n, seed=spec.seed + seed_offset)


def time_oracle(wl, k8=None):
    """One oracle call over the workload (over int8 codes k8 = (codes, scales)
    if given); seconds."""
    import oracle
    q, k, v = wl.q.numpy(), wl.k_pool.numpy(), wl.v_pool.numpy()
    t0 = time.perf_counter()
    if k8 is None:
        oracle.paged_attention(q, k, v, wl.block_tables, wl.lens, scale=wl.scale,
                               q_len=wl.q.shape[1])
    else:
        oracle.paged_attention_q8k(q, k8[0], k8[1], v, wl.block_tables, wl.lens, scale=wl.scale,
                                   q_len=wl.q.shape[1])
    return time.perf_counter() - t0


def host_copy(wl):
    """The workload's inputs as host arrays: only the blocks the tables use,
    renumbered (plain data movement)."""
    import numpy as np
    import torch
    tables = wl.block_tables
    ids = np.unique(tables[tables >= 0])
    idx = torch.as_tensor(ids, device=wl.k_pool.device, dtype=torch.long)
    K = wl.k_pool[idx].cpu().numpy()
    V = wl.v_pool[idx].cpu().numpy()
    t2 = np.where(tables >= 0, np.searchsorted(ids, np.maximum(tables, 0)), -1).astype(np.int32)
    return wl.q.cpu().numpy(), K, V, t2


def cpu_model():
    """The host CPU's model name (from /proc/cpuinfo), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def cpu_baseline(wl, target_s, q8k=False):
    """The oracle, as it stands, over the whole workload of this run (its
    sequences, blocks and queries copied to the host; int8 K codes made by
    the oracle's own quantiser), repeated until about target_s seconds of CPU
    time have been spent, on all host threads; then on one thread over the
    first sequences of the same workload (about target_s / 2 seconds)."""
    import numpy as np
    import oracle
    q, K, V, t2 = host_copy(wl)
    s = wl.spec
    K8 = sc = None
    if q8k:
        K8, sc = quantise_pool_host(K)

    def call(nseq):
        if q8k:
            oracle.paged_attention_q8k(q[:nseq], K8, sc, V, t2[:nseq], wl.lens[:nseq],
                                       scale=wl.scale, q_len=q.shape[1])
        else:
            oracle.paged_attention(q[:nseq], K, V, t2[:nseq], wl.lens[:nseq], scale=wl.scale,
                                   q_len=q.shape[1])

    def kvb(nseq):
        return algorithmic_bytes(wl.lens[:nseq], q.shape[2], s.Hkv, q.shape[3], s.bs, q.shape[1],
                                 1 if q8k else 2)[0]

    B = int(wl.lens.shape[0])
    reps, spent = 0, 0.0
    while reps == 0 or spent < target_s:
        t0 = time.perf_counter()
        call(B)
        spent += time.perf_counter() - t0
        reps += 1
    threads = oracle.num_threads()
    res = {"value": round(kvb(B) * reps / spent / 1e9, 4), "unit": "GB/s", "cores": threads,
           "kind": "oracle", "cpu_model": cpu_model(),
           "sample": f"whole workload of this run ({B} sequences, {int(wl.lens.sum())} "
                     f"tokens) x {reps} repeat(s), fp64 C oracle, {spent:.2f} s"}
    # one thread: as many leading sequences as fit in about target_s / 2
    per_seq = spent / reps / B * threads
    n1 = int(max(1, min(B, (target_s / 2) / max(per_seq, 1e-6))))
    oracle.set_num_threads(1)
    try:
        t0 = time.perf_counter()
        call(n1)
        t1 = time.perf_counter() - t0
    finally:
        oracle.set_num_threads(threads)
    res["single_thread"] = {"value": round(kvb(n1) / t1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                            "sample": f"first {n1} of {B} sequences "
                                      f"({int(np.sum(wl.lens[:n1]))} tokens), {t1:.2f} s"}
    return res


def run_reference(args):
    import oracle
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    from workloads.synth import CONFIGS
    base, q8k = split_workload(args.workload)
    spec = CONFIGS[base]
    if spec.q_len > 32:
        return run_reference_prefill(args, base, spec, world)
    per_step = max(0.2, min(2.0, 120.0 / max(1, args.steps + args.warmup)))
    wl = oracle_sample(args.workload, per_step)
    k8 = quantise_pool_host(wl.k_pool.numpy()) if q8k else None
    for _ in range(args.warmup):
        time_oracle(wl, k8)
    times = [time_oracle(wl, k8) for _ in range(args.steps)]
    kvb = algorithmic_bytes(wl.lens, spec.Hq, spec.Hkv, spec.D, spec.bs, spec.q_len,
                            1 if q8k else 2)[0]
    total = sum(times)
    value = kvb * args.steps / total / 1e9
    sample = (f"{wl.B} of {spec.B} sequences of {args.workload} per step (same length recipe), "
              f"{int(wl.lens.sum())} tokens, fp64 C oracle")
    return {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": args.workload, "description": spec.description},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "kind": "oracle",
                             "cores": oracle.num_threads(), "cpu_model": cpu_model(),
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def run_reference_prefill(args, base, spec, world):
    """The oracle on a bounded window of the chunked-prefill workload: the
    first 16 positions of one sequence's chunk per step."""
    import oracle
    from workloads import make_workload
    wl = make_workload(base, "cpu", B=1, seed=spec.seed)
    n_pos = 16
    q, K, V, t2, lens = prefill_window(wl, spec.q_len, 1, n_pos)

    def once():
        t0 = time.perf_counter()
        oracle.paged_attention(q, K, V, t2, lens, scale=wl.scale, q_len=n_pos)
        return time.perf_counter() - t0
    for _ in range(args.warmup):
        once()
    times = [once() for _ in range(args.steps)]
    fl = prefill_flops(lens, spec.Hq, spec.D, n_pos) * args.steps
    value = fl / sum(times) / 1e12
    sample = (f"first {n_pos} positions of one sequence's {spec.q_len}-token chunk per step "
              f"({int(lens[0])} tokens, {spec.Hq} heads), fp64 C oracle")
    return {"metric": "paged prefill attention TFLOP/s", "value": round(value, 6), "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(sum(times) / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": {"workload": args.workload, "description": spec.description},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "kind": "oracle",
                             "cores": oracle.num_threads(), "cpu_model": cpu_model(),
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main(argv=None):
    global CONSUMER
    args = parse_args(argv)
    CONSUMER = args.consumer
    from workloads.synth import CONFIGS
    if args.impl == "reference":
        res = run_reference(args)
    elif CONFIGS[split_workload(args.workload)[0]].q_len > 32:
        res = run_prefill(args)
    else:
        res = run_ours(args)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
