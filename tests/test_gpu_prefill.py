"""Paged chunked prefill (tcgen05 tensor cores) vs the fp64 oracle (needs a B200).

Same tolerance as decode: |gpu - ref| <= 2e-3 + 1e-2 |ref|.  Cases span
several 128-row query tiles, ragged last tiles, GQA groups 1 / 4 / 8 / 16,
8- and 16-token blocks, prefixes that end inside a block, and chunks that are
the whole sequence.
"""
import numpy as np
import pytest
import torch

from paged_helpers import assert_close, device_inputs, oracle_subset
from workloads import make_workload

pytestmark = pytest.mark.gpu

pkv = pytest.importorskip("paged_kv_cache_371_b200")


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    pkv.device_error(reset=True)
    yield
    torch.cuda.synchronize()


@pytest.mark.parametrize("Hq,Hkv,bs,q_len,lens", [
    (8, 8, 16, 37, [37, 100]),            # MHA rows, whole-sequence chunk and a prefix
    (32, 8, 16, 64, [64, 200, 1031]),     # G=4: 16 positions per tile, 4 tiles
    (64, 8, 16, 48, [300, 48, 777]),      # G=8: 16 positions per tile, ragged last tile
    (16, 1, 8, 24, [24, 95, 513]),        # G=16, 8-token blocks
    (8, 8, 8, 200, [200, 333]),           # MHA, 2 tiles of 128 positions
])
def test_prefill_full_compare(Hq, Hkv, bs, q_len, lens):
    wl = make_workload("llama70b_gqa", "cuda", lens=np.array(lens, np.int32), bs=bs, q_len=q_len,
                       Hq=Hq, Hkv=Hkv, D=128, seed=q_len + Hq)
    bt, cl = device_inputs(wl)
    out = pkv.paged_prefill_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale, q_len)
    torch.cuda.synchronize()
    assert pkv.device_error() == 0
    ref = oracle_subset(wl, list(range(wl.B)), q_len=q_len)
    assert_close(out, ref, f"prefill Hq{Hq} Hkv{Hkv} bs{bs} q{q_len}")


def test_prefill_matches_verify_for_short_windows():
    """A 5-token window through prefill and through the verify path agree."""
    wl = make_workload("long_verify", "cuda", B=2, max_len=3000)
    bt, cl = device_inputs(wl)
    a = pkv.paged_prefill_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale, 5)
    b = pkv.paged_verify_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale, 5)
    ref = oracle_subset(wl, [0, 1], q_len=5)
    assert_close(a, ref, "prefill")
    assert_close(b, ref, "verify")


def _stage_max_jumps(wl, s, q_len, stage=128):
    """log2-unit growth of each row's running score maximum at the start of
    every later stage, from the inputs (fp64): used to show that a case
    really makes the maximum jump after the first stage."""
    bs = wl.k_pool.shape[2]
    L = int(wl.lens[s])
    n = -(-L // bs)
    ids = torch.as_tensor(wl.block_tables[s, :n].astype(np.int64), device=wl.k_pool.device)
    K = wl.k_pool[ids].double().permute(1, 0, 2, 3).reshape(wl.k_pool.shape[1], n * bs, -1)[:, :L]
    q = wl.q[s].double()                                   # [q_len][Hq][D]
    G = q.shape[1] // K.shape[0]
    sc = torch.einsum("jhd,htd->jht", q, K.repeat_interleave(G, 0)) * wl.scale / np.log(2.0)
    pos = torch.arange(L, device=sc.device)
    lim = L - q_len + torch.arange(q_len, device=sc.device)
    sc = sc.masked_fill(pos[None, None, :] > lim[:, None, None], float("-inf"))
    best = 0.0
    m = sc[:, :, :stage].amax(-1)
    for t0 in range(stage, L, stage):
        mn = torch.maximum(m, sc[:, :, t0:t0 + stage].amax(-1))
        best = max(best, float((mn - m)[torch.isfinite(m)].max()))
        m = mn
    return best


@pytest.mark.parametrize("Hq,Hkv,bs,q_len,lens", [
    (8, 8, 16, 200, [1031, 700]),      # MHA rows, 16-token blocks
    (64, 8, 8, 48, [1100, 600]),       # G=8, 8-token blocks
    (64, 8, 16, 160, [900, 1200]),     # G=8, 16-token blocks, two tiles per CTA
])
def test_prefill_planted_late_maxima(Hq, Hkv, bs, q_len, lens):
    """Keys aligned with the queries planted in stage 1, stage 3 and the last
    (partial) stage, each dominating everything before it by > 2^8 in weight:
    every stage-j >= 1 rescale of O in tensor memory runs, and the output
    must still be the oracle's."""
    from planted import plant
    wl = make_workload("llama70b_gqa", "cuda", lens=np.array(lens, np.int32), bs=bs, q_len=q_len,
                       Hq=Hq, Hkv=Hkv, D=128, seed=q_len + 7 * Hq)
    plan = {}
    for s, L in enumerate(lens):
        plan[s] = [(200, 40.0), (450, 80.0), (L - q_len + 5, 120.0), (L - 2, 160.0)]
    plant(wl, plan, seed=q_len)
    assert _stage_max_jumps(wl, 0, q_len) > 8.0
    bt, cl = device_inputs(wl)
    out = pkv.paged_prefill_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale, q_len)
    torch.cuda.synchronize()
    assert pkv.device_error() == 0
    ref = oracle_subset(wl, list(range(wl.B)), q_len=q_len)
    assert_close(out, ref, f"planted prefill Hq{Hq} Hkv{Hkv} bs{bs}")


@pytest.mark.parametrize("Hq,Hkv,bs", [(8, 8, 16), (64, 8, 8), (64, 8, 16)])
def test_prefill_ramped_keys(Hq, Hkv, bs):
    """Key norms growing along the context (x(1 + t/150)): the row maxima
    climb stage after stage and the lazy rescale fires repeatedly."""
    from planted import ramp
    q_len = 96
    lens = [1000, 777]
    wl = make_workload("llama70b_gqa", "cuda", lens=np.array(lens, np.int32), bs=bs, q_len=q_len,
                       Hq=Hq, Hkv=Hkv, D=128, seed=5 + Hq + bs)
    ramp(wl, 150.0)
    assert _stage_max_jumps(wl, 0, q_len) > 2.0
    bt, cl = device_inputs(wl)
    out = pkv.paged_prefill_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale, q_len)
    torch.cuda.synchronize()
    assert pkv.device_error() == 0
    ref = oracle_subset(wl, list(range(wl.B)), q_len=q_len)
    assert_close(out, ref, f"ramped prefill Hq{Hq} bs{bs}")


def test_prefill_chunk_full_size_whole_sequences():
    """The benchmark's chunked-prefill workload at full size (8 sequences, a
    512-token chunk each on prefixes of 1-4K tokens, GQA 64/8), launched as
    the benchmark launches it; every row of every head of the shortest and
    the longest sequence compared with the oracle."""
    wl = make_workload("prefill_chunk", "cuda")
    q_len = wl.spec.q_len
    bt, cl = device_inputs(wl)
    out = pkv.paged_prefill_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale, q_len)
    torch.cuda.synchronize()
    assert pkv.device_error() == 0
    seqs = sorted({int(np.argmin(wl.lens)), int(np.argmax(wl.lens))})
    ref = oracle_subset(wl, seqs, q_len=q_len)
    assert_close(out[torch.as_tensor(seqs, device="cuda")], ref, "prefill_chunk full size")


def test_prefill_loader_wait_limit_times_out_and_recovers():
    """Failure detection without a fault: a 1 ns limit on the prefill loader's
    wait for a free K/V slot makes it give up after the first stages; the MMA
    and softmax warps reach their own bounded waits, tensor memory is
    released, the call returns with KV_DEV_TIMEOUT in the device error word,
    and the next ordinary launch is correct."""
    import time
    wl = make_workload("llama70b_gqa", "cuda", lens=np.array([1500, 900], np.int32), q_len=64,
                       Hq=64, Hkv=8, D=128, seed=3)
    bt, cl = device_inputs(wl)
    pkv.paged_prefill_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale, 64)  # warm
    assert pkv.device_error() == 0
    t0 = time.perf_counter()
    pkv.paged_prefill_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale, 64, producer_wait_ns=1)
    err = pkv.device_error()
    dt = time.perf_counter() - t0
    assert err & pkv._abi.KV_DEV_TIMEOUT
    assert dt < 20.0, f"a timed-out launch took {dt:.1f} s"
    out = pkv.paged_prefill_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale, 64)
    torch.cuda.synchronize()
    assert pkv.device_error() == 0
    assert_close(out, oracle_subset(wl, [0, 1], q_len=64), "prefill after a timeout")
