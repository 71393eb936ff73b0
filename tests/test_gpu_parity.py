"""CUDA path vs the fp64 oracle on the same seeded inputs (needs a B200).

Attention: |gpu - ref| <= 2e-3 + 1e-2 |ref| elementwise; append, block copy
and all bookkeeping: bit-exact.  Full-size configs run in the launch
configuration the benchmark times and are checked on every sequence;
smaller cases (forced context splits, planted late maxima, edge cases) are
checked in full.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle.block_spec import BlockPoolSpec
from paged_helpers import assert_close, device_inputs, oracle_subset
from workloads import make_workload, normal_fp16, random_distinct_slots

pytestmark = pytest.mark.gpu

pkv = pytest.importorskip("paged_kv_cache_371_b200")


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    pkv.device_error(reset=True)
    yield
    torch.cuda.synchronize()


def _u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


# ----------------------------------------------------------------------------- append / copy

@pytest.mark.parametrize("shape", [(16, 4, 16, 64, 2), (300, 8, 16, 128, 128), (97, 8, 8, 128, 33)])
def test_append_bit_exact(shape):
    nb, Hkv, bs, D, T = shape
    K = normal_fp16((nb, Hkv, bs, D), 11, "cuda")
    V = normal_fp16((nb, Hkv, bs, D), 12, "cuda")
    kn = normal_fp16((T, Hkv, D), 13, "cuda")
    vn = normal_fp16((T, Hkv, D), 14, "cuda")
    slots = random_distinct_slots(T, nb * bs, 15)
    slots[::5] = -1  # padding tokens
    ref_k, ref_v = oracle.append(K.cpu().numpy(), V.cpu().numpy(), kn.cpu().numpy(),
                                 vn.cpu().numpy(), slots)
    pkv.paged_kv_append(kn, vn, torch.as_tensor(slots, device="cuda"), K, V)
    assert pkv.device_error() == 0
    assert np.array_equal(_u16(K), ref_k.view(np.uint16))
    assert np.array_equal(_u16(V), ref_v.view(np.uint16))


def test_append_bad_slot_is_flagged_and_skipped():
    nb, Hkv, bs, D = 8, 2, 16, 64
    K = normal_fp16((nb, Hkv, bs, D), 1, "cuda")
    V = normal_fp16((nb, Hkv, bs, D), 2, "cuda")
    K0, V0 = K.clone(), V.clone()
    kn = normal_fp16((2, Hkv, D), 3, "cuda")
    slots = torch.tensor([nb * bs, 3], dtype=torch.int64, device="cuda")
    pkv.paged_kv_append(kn, kn, slots, K, V)
    err = pkv.device_error()
    assert err & pkv._abi.KV_DEV_BAD_SLOT
    assert torch.equal(K.view(torch.int16)[0, :, 3], kn.view(torch.int16)[1])
    K[0, :, 3] = K0[0, :, 3]
    V[0, :, 3] = V0[0, :, 3]
    assert torch.equal(K.view(torch.int16), K0.view(torch.int16))


def test_copy_blocks_bit_exact():
    nb, Hkv, bs, D = 64, 8, 16, 128
    K = normal_fp16((nb, Hkv, bs, D), 21, "cuda")
    V = normal_fp16((nb, Hkv, bs, D), 22, "cuda")
    rng = np.random.Generator(np.random.PCG64(23))
    perm = rng.permutation(nb)
    pairs = np.stack([perm[:10], perm[10:20]], 1).astype(np.int32)
    ref_k, ref_v = oracle.copy_blocks(K.cpu().numpy(), V.cpu().numpy(), pairs)
    pkv.paged_kv_copy_blocks(K, V, torch.as_tensor(pairs, device="cuda"))
    assert pkv.device_error() == 0
    assert np.array_equal(_u16(K), ref_k.view(np.uint16))
    assert np.array_equal(_u16(V), ref_v.view(np.uint16))


# ----------------------------------------------------------------------------- decode / verify

def _run(wl, q_len=1, **kw):
    bt, cl = device_inputs(wl)
    if kw:
        out = pkv.paged_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale, q_len=q_len, **kw)
    elif q_len == 1:
        out = pkv.paged_decode_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale)
    else:
        out = pkv.paged_verify_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale, q_len)
    assert pkv.device_error() == 0
    return out


@pytest.mark.parametrize("name", ["llama7b_mha", "llama70b_gqa", "llama70b_gqa_bs8", "prefix_beam",
                                  "long_decode", "long_verify"])
def test_full_size_config_every_sequence(name):
    """Each decode config at full size, in the launch configuration the
    benchmark times: every output element of every sequence (so every CTA's
    split boundary and every merged row of the real partition) against the
    oracle."""
    wl = make_workload(name, "cuda")
    q_len = wl.spec.q_len
    out = _run(wl, q_len)
    ref = oracle_subset(wl, list(range(wl.B)), q_len)
    assert_close(out, ref, name)


@pytest.mark.parametrize("Hq,Hkv,bs,q_len", [
    (8, 8, 16, 1),      # one row per KV head: FMA path
    (64, 8, 16, 1),     # GQA 8: tensor cores, one m16 row tile
    (64, 8, 8, 1),      # the same with 8-token blocks
    (32, 8, 16, 5),     # verify window of 5 x 4 heads: two m16 row tiles
])
@pytest.mark.parametrize("grid,min_split", [(0, 0), (300, 1), (7, 1)])
def test_decode_planted_late_maxima(Hq, Hkv, bs, q_len, grid, min_split):
    """Keys aligned with the queries planted after the first stage, each
    dominating everything before it: the running maximum jumps several
    times inside one CTA's run and across split boundaries, so the rescale
    of the partial output (and the split merge) carry the result."""
    from planted import plant
    lens = np.array([1500, 700, 333], np.int32)
    wl = make_workload("llama70b_gqa", "cuda", lens=lens, bs=bs, q_len=q_len, Hq=Hq, Hkv=Hkv, D=128,
                       seed=11 + Hq + bs + q_len)
    plan = {s: [(70, 40.0), (300, 80.0), (int(L) - 10, 120.0), (int(L) - 1, 160.0)]
            for s, L in enumerate(lens)}
    plant(wl, plan, seed=Hq + q_len)
    out = _run(wl, q_len, grid_ctas=grid, min_split_blocks=min_split)
    ref = oracle_subset(wl, list(range(wl.B)), q_len)
    assert_close(out, ref, f"planted Hq{Hq} Hkv{Hkv} bs{bs} q{q_len} grid{grid}")


@pytest.mark.parametrize("name,kw", [("long_decode", {"B": 4}), ("llama7b_mha", {"B": 16}),
                                     ("long_verify", {"B": 4})])
def test_loader_wait_limit_times_out_and_recovers(name, kw):
    """Failure detection without a fault: a 1 ns limit on the loading warp's
    waits for a free stage makes it give up; the CTAs finish the stages
    already loaded and stop, the call returns promptly with KV_DEV_TIMEOUT
    in the device error word, and the next ordinary launch is correct."""
    import time
    wl = make_workload(name, "cuda", **kw)
    q_len = wl.spec.q_len
    bt, cl = device_inputs(wl)
    _run(wl, q_len)  # warm: tensor maps and kernel attributes set up
    t0 = time.perf_counter()
    pkv.paged_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale, q_len=q_len,
                        producer_wait_ns=1)
    err = pkv.device_error()
    dt = time.perf_counter() - t0
    assert err & pkv._abi.KV_DEV_TIMEOUT
    assert dt < 1.0, f"a timed-out launch took {dt:.2f} s"
    out = _run(wl, q_len)
    seqs = [0, wl.B - 1]
    assert_close(out[torch.as_tensor(seqs, device="cuda")], oracle_subset(wl, seqs, q_len), name)


def test_tiny_config_full_with_append():
    """Config 1: decode, then append one token per sequence through the block
    manager and the append kernel, then decode again."""
    wl = make_workload("tiny", "cuda")
    out = _run(wl)
    assert_close(out, oracle_subset(wl, [0, 1]), "tiny")

    bs = wl.spec.bs
    cap = wl.block_tables.shape[1] + 1
    impl = pkv.KVPool(wl.num_blocks, bs, order=wl.order)
    spec = BlockPoolSpec(wl.num_blocks, bs, wl.order)
    tables = np.full((wl.B, cap), -1, np.int32)
    nblk = np.zeros(wl.B, np.int32)
    spec_tables = [[] for _ in range(wl.B)]
    for s in range(wl.B):  # rebuild the existing sequences token by token
        for t in range(int(wl.lens[s])):
            spec.reserve_slot(spec_tables[s], t)
            nblk[s] = impl.reserve_slot(tables[s], int(nblk[s]), t)[1]
        assert tables[s, :nblk[s]].tolist() == wl.block_tables[s][wl.block_tables[s] >= 0].tolist()
    slots, pairs = impl.reserve_slots(tables, nblk, wl.lens)
    spec_slots = [spec.reserve_slot(spec_tables[s], int(wl.lens[s]))[1] for s in range(wl.B)]
    assert slots.tolist() == spec_slots and len(pairs) == 0
    Hkv, D = wl.spec.Hkv, wl.spec.D
    kn = normal_fp16((wl.B, Hkv, D), 31, "cuda")
    vn = normal_fp16((wl.B, Hkv, D), 32, "cuda")
    ref_k, ref_v = oracle.append(wl.k_pool.cpu().numpy(), wl.v_pool.cpu().numpy(),
                                 kn.cpu().numpy(), vn.cpu().numpy(), np.array(spec_slots))
    pkv.paged_kv_append(kn, vn, torch.as_tensor(slots, device="cuda"), wl.k_pool, wl.v_pool)
    assert np.array_equal(_u16(wl.k_pool), ref_k.view(np.uint16))
    new_lens = (wl.lens + 1).astype(np.int32)
    bt = torch.as_tensor(tables, device="cuda")
    out2 = pkv.paged_decode_attention(wl.q, wl.k_pool, wl.v_pool, bt,
                                      torch.as_tensor(new_lens, device="cuda"), wl.scale)
    spec_tab = np.full((wl.B, cap), -1, np.int32)
    for s in range(wl.B):
        spec_tab[s, :len(spec_tables[s])] = spec_tables[s]
    ref2 = oracle.paged_attention(wl.q.cpu().numpy(), ref_k, ref_v, spec_tab, new_lens,
                                  scale=wl.scale)
    assert_close(out2, ref2, "tiny after append")


@pytest.mark.parametrize("bs,int8_k,G", [(8, False, 8), (8, True, 8), (16, True, 8), (16, True, 1),
                                          (8, True, 1), (16, True, 4)])
@pytest.mark.parametrize("Hkv", [2, 8])
@pytest.mark.parametrize("grid,min_split", [(0, 0), (300, 1), (7, 1)])
def test_head_pairs(Hkv, grid, min_split, bs, int8_k, G):
    """8-token blocks with GQA groups of 8, or int8 keys with groups of 8, 4
    or 1 (MHA), one query per sequence: each staged tile holds two adjacent
    KV heads of a block (one copy), and row tile h (padded rows 8h ..)
    reads head h's rows (and, over int8 keys, head h's channel scales).  Each
    head's queries and planted keys follow their own direction, so taking a
    row tile's keys, values, scales or queries from the other head of the
    pair moves the outputs far from the oracle's."""
    from planted import plant
    lens = np.array([0, 1, 7, 8, 9, 64, 65, 333, 1500], np.int32)
    wl = make_workload("llama70b_gqa", "cuda", lens=lens, bs=bs, q_len=1, Hq=G * Hkv, Hkv=Hkv, D=128,
                       seed=90 + Hkv + bs + G)
    plan = {s: [(int(L) // 3, 60.0), (int(L) - 1, 120.0)] for s, L in enumerate(lens) if L > 3}
    plant(wl, plan, seed=13 + Hkv)
    if int8_k:
        from test_gpu_q8k import _oracle_subset_q8k, _pool_scales, _quantise_on_device
        scales = _pool_scales(wl)
        kq, vq, sc = _quantise_on_device(wl, scales)
        bt, cl = device_inputs(wl)
        out = pkv.paged_attention_q8k(wl.q, kq, sc, vq, bt, cl, wl.scale, q_len=1, grid_ctas=grid,
                                      min_split_blocks=min_split)
        torch.cuda.synchronize()
        assert pkv.device_error() == 0
        ref = _oracle_subset_q8k(wl, kq, scales, np.arange(wl.B), wl.q, 1)
    else:
        out = _run(wl, 1, grid_ctas=grid, min_split_blocks=min_split)
        torch.cuda.synchronize()
        ref = oracle_subset(wl, list(range(wl.B)))
    assert_close(out, ref, f"head pairs bs{bs} G{G} Hkv{Hkv} grid{grid} int8 {int8_k}")
    assert not out[0].any()  # an empty context gives zeros


@pytest.mark.parametrize("name,B", [("llama70b_gqa", 64), ("llama7b_mha", 32)])
def test_attention_launched_behind_the_append_reads_the_new_token(name, B):
    """The attention launch may start its set-up while the append just before
    it in the stream still runs (programmatic dependent launch); its loader
    must wait for the append before reading the pools.  Each sequence appends
    a key aligned with its queries, dominating every other score, into a slot
    that held NaN: a read before the append lands gives NaN or a far-off
    output, a correct one gives (nearly) the new token's V."""
    from workloads import CONFIGS
    rng = np.random.Generator(np.random.PCG64(B))
    bs = CONFIGS[name].bs
    lens = rng.integers(100, 900, size=B).astype(np.int32)
    lens[lens % bs == 0] += 1                      # room left in each last block
    wl = make_workload(name, "cuda", lens=lens, seed=61 + B)
    Hkv, D = wl.k_pool.shape[1], wl.k_pool.shape[3]
    G = wl.q.shape[2] // Hkv
    # the queries of each (sequence, kv head) share a direction u; the new key is 100 u
    g = torch.Generator(device="cpu")
    g.manual_seed(5)
    u = torch.randn((B, Hkv, D), generator=g, dtype=torch.float64)
    u /= u.norm(dim=-1, keepdim=True)
    q = 0.5 * wl.q.double().cpu() + 4.0 * u.repeat_interleave(G, dim=1)[:, None, :, :]
    wl.q = q.to(torch.float16).cuda()
    k_new = (100.0 * u).to(torch.float16)
    v_new = normal_fp16((B, Hkv, D), 62, "cpu")
    blk = np.array([wl.block_tables[s, lens[s] // bs] for s in range(B)], np.int64)
    off = (lens % bs).astype(np.int64)
    slots = blk * bs + off
    k0, v0 = wl.k_pool.cpu().numpy(), wl.v_pool.cpu().numpy()
    assert np.isnan(k0[blk, :, off, :]).all() and np.isnan(v0[blk, :, off, :]).all()
    ref_k, ref_v = oracle.append(k0, v0, k_new.numpy(), v_new.numpy(), slots)
    new_lens = (lens + 1).astype(np.int32)
    # every device input in place before the two launches, which run back to back
    kd, vd, sd = k_new.cuda(), v_new.cuda(), torch.as_tensor(slots, device="cuda")
    bt = torch.as_tensor(wl.block_tables, device="cuda")
    cl = torch.as_tensor(new_lens, device="cuda")
    out = torch.empty_like(wl.q)
    torch.cuda.synchronize()
    pkv.paged_kv_append(kd, vd, sd, wl.k_pool, wl.v_pool)
    pkv.paged_decode_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale, out=out)
    torch.cuda.synchronize()
    assert pkv.device_error() == 0
    ref = oracle.paged_attention(wl.q.cpu().numpy(), ref_k, ref_v, wl.block_tables, new_lens,
                                 scale=wl.scale)
    assert_close(out, ref, f"{name} behind the append")
    want = v_new.repeat_interleave(G, dim=1).double().numpy()
    assert np.abs(out[:, 0].cpu().double().numpy() - want).max() < 0.02


@pytest.mark.parametrize("Hq,Hkv,D,bs,q_len", [
    (4, 4, 64, 16, 1), (8, 8, 128, 8, 1),           # FMA path (one row per KV head)
    (8, 2, 64, 16, 1), (64, 8, 128, 16, 1),          # tensor-core path, one m16 tile
    (32, 8, 128, 8, 5), (16, 2, 128, 16, 4),         # verify windows, two m16 tiles
    (4, 4, 128, 16, 3), (6, 2, 64, 8, 1)])
@pytest.mark.parametrize("grid,min_split", [(0, 0), (300, 1), (7, 1)])
def test_forced_splits_full_compare(Hq, Hkv, D, bs, q_len, grid, min_split):
    """Oracle-sized problems over several tiles and ragged tails, with the
    context split across many CTAs (merge path) or few CTAs (long runs)."""
    rng = np.random.Generator(np.random.PCG64(Hq * 131 + D + bs + q_len))
    B = 5
    lens = np.array([1, bs, 3 * bs + 1, 200, 411], dtype=np.int32)
    lens = np.maximum(lens, q_len)
    wl = make_workload("llama70b_gqa", "cuda", lens=lens, bs=bs, q_len=q_len, Hq=Hq, Hkv=Hkv, D=D,
                       seed=int(rng.integers(1 << 30)))
    out = _run(wl, q_len, grid_ctas=grid, min_split_blocks=min_split)
    ref = oracle_subset(wl, list(range(B)), q_len)
    assert_close(out, ref, f"Hq{Hq} Hkv{Hkv} D{D} bs{bs} q{q_len} grid{grid}")


@pytest.mark.parametrize("seg_cost", [-1, 1, 4, 13])
@pytest.mark.parametrize("grid", [0, 61])
@pytest.mark.parametrize("Hq,Hkv", [(16, 4), (8, 8)])  # tensor-core path, FMA path
def test_segment_cost_partition(seg_cost, grid, Hq, Hkv):
    """Many short sequences: CTA runs that start or end inside a segment's
    virtual cost units, splits and merges all give the oracle's result."""
    rng = np.random.Generator(np.random.PCG64(17))
    lens = rng.integers(1, 300, size=40).astype(np.int32)
    wl = make_workload("llama70b_gqa", "cuda", lens=lens, seed=19, Hq=Hq, Hkv=Hkv, D=128)
    out = _run(wl, 1, grid_ctas=grid, min_split_blocks=1, seg_cost_blocks=seg_cost)
    assert_close(out, oracle_subset(wl, list(range(wl.B))), f"Hq{Hq} Hkv{Hkv} seg_cost {seg_cost} grid {grid}")


@pytest.mark.parametrize("B,Hq,Hkv,maxlen,grid", [
    (700, 8, 2, 90, 0),      # > 256 sequences: the device scan loops over chunks
    (300, 32, 1, 400, 37),   # MQA: 32 query rows per KV head (the largest supported)
    (1, 16, 4, 131072, 0),   # one 128K-token sequence split across every CTA
])
def test_scale_edges(B, Hq, Hkv, maxlen, grid):
    rng = np.random.Generator(np.random.PCG64(B + Hq))
    lens = rng.integers(1, maxlen + 1, size=B).astype(np.int32) if B > 1 else np.array([maxlen], np.int32)
    wl = make_workload("llama70b_gqa", "cuda", lens=lens, seed=23, Hq=Hq, Hkv=Hkv, D=128)
    out = _run(wl, 1, grid_ctas=grid) if grid else _run(wl)
    assert_close(out, oracle_subset(wl, list(range(wl.B))), f"B{B} Hkv{Hkv}")


def test_empty_batch_is_a_no_op():
    wl = make_workload("tiny", "cuda")
    bt = torch.zeros((0, 4), dtype=torch.int32, device="cuda")
    cl = torch.zeros((0,), dtype=torch.int32, device="cuda")
    q = torch.zeros((0, 1, 4, 64), dtype=torch.float16, device="cuda")
    out = pkv.paged_decode_attention(q, wl.k_pool, wl.v_pool, bt, cl, wl.scale)
    assert out.shape == (0, 1, 4, 64) and pkv.device_error() == 0


def test_edge_cases():
    """Empty context (zeros), one token (exactly V), exact block multiples,
    a window longer than the context (zeros for rows that see nothing)."""
    lens = np.array([0, 1, 16, 17, 32, 2], dtype=np.int32)
    wl = make_workload("llama70b_gqa", "cuda", lens=lens, q_len=1, seed=77, Hq=8, Hkv=2, D=128)
    out = _run(wl, 1, grid_ctas=5, min_split_blocks=1)
    ref = oracle_subset(wl, list(range(len(lens))))
    assert_close(out, ref, "edge decode")
    assert not out[0].any()
    # one token: softmax weight exactly 1, output bit-exactly V (fp16)
    v0 = wl.v_pool[int(wl.block_tables[1, 0]), :, 0, :]  # [Hkv][D]
    G = 8 // 2
    exp = v0.repeat_interleave(G, dim=0)
    assert torch.equal(out[1, 0].view(torch.int16), exp.view(torch.int16))
    # verify window of 3 over contexts of 2 and 1 tokens: rows past the context see nothing
    wl.q = normal_fp16((len(lens), 3, 8, 128), 5, "cuda")
    out3 = _run(wl, 3, grid_ctas=3)
    ref3 = oracle_subset(wl, list(range(len(lens))), q_len=3)
    assert_close(out3, ref3, "edge verify")


def test_permutation_invariance_bit_exact():
    """Moving blocks to other physical ids (same work split) changes no bit."""
    wl = make_workload("llama70b_gqa", "cuda", B=24, max_len=700, seed=5)
    out = _run(wl).clone()
    rng = np.random.Generator(np.random.PCG64(6))
    perm = rng.permutation(wl.num_blocks)
    pt = torch.as_tensor(perm, device="cuda", dtype=torch.long)
    k2 = torch.empty_like(wl.k_pool)
    v2 = torch.empty_like(wl.v_pool)
    k2[pt] = wl.k_pool
    v2[pt] = wl.v_pool
    t2 = np.where(wl.block_tables >= 0, perm[np.maximum(wl.block_tables, 0)], -1).astype(np.int32)
    wl.k_pool, wl.v_pool, wl.block_tables = k2, v2, t2
    out2 = _run(wl)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


@pytest.mark.parametrize("name,kw", [("llama70b_gqa_bs8", {"B": 40, "max_len": 900}),
                                     ("llama7b_mha", {"B": 12, "max_len": 1500}),
                                     ("long_verify", {"B": 2, "max_len": 3000})])
def test_deterministic_across_runs_and_splits(name, kw):
    """Same inputs and launch -> the same bits; a different split of the
    context -> within tolerance of the first."""
    wl = make_workload(name, "cuda", **kw)
    q_len = wl.spec.q_len
    a = _run(wl, q_len).clone()
    b = _run(wl, q_len).clone()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    c = _run(wl, q_len, grid_ctas=37, min_split_blocks=3)
    ref = oracle_subset(wl, list(range(wl.B)), q_len)
    assert_close(a, ref, name)
    assert_close(c, ref, name + " resplit")


def test_bad_block_id_is_flagged_without_fault():
    wl = make_workload("llama70b_gqa", "cuda", B=6, max_len=300, seed=8)
    wl.block_tables[2, 1] = wl.num_blocks + 5
    bt, cl = device_inputs(wl)
    out = pkv.paged_decode_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale)
    err = pkv.device_error()
    assert err & pkv._abi.KV_DEV_BAD_BLOCK
    others = [0, 1, 3, 4, 5]
    assert_close(out[torch.as_tensor(others, device="cuda")], oracle_subset(wl, others),
                 "untouched sequences")


# ----------------------------------------------------------------------------- prefix + beams

@pytest.mark.parametrize("fork_len", [1024, 1030])
def test_prefix_sharing_and_beam_copy_on_write(fork_len):
    """Config 4: 64 requests share a 2048-token prefix (refcount 64); 4 beams
    forked at fork_len each append one token; a shared partial last block is
    copied on write.  Bookkeeping and pools bit-exact, attention within
    tolerance."""
    wl = make_workload("prefix_beam", "cuda", spare_blocks=600)
    bs, Hkv, D = wl.spec.bs, wl.spec.Hkv, wl.spec.D
    nb = wl.num_blocks
    cap = wl.block_tables.shape[1] + 2
    impl = pkv.KVPool(nb, bs, order=wl.order)
    spec = BlockPoolSpec(nb, bs, wl.order)
    P = wl.extra["prefix_blocks"]
    # request 0 builds the prefix, the others fork it, then each grows its suffix
    t_impl = np.full((wl.B, cap), -1, np.int32)
    n_impl = np.zeros(wl.B, np.int32)
    t_spec = [[] for _ in range(wl.B)]
    for t in range(P * bs):
        spec.reserve_slot(t_spec[0], t)
        n_impl[0] = impl.reserve_slot(t_impl[0], int(n_impl[0]), t)[1]
    for s in range(1, wl.B):
        spec.fork(t_spec[0][:P])
        impl.fork(t_impl[0, :P])
        t_spec[s] = list(t_spec[0][:P])
        t_impl[s, :P] = t_impl[0, :P]
        n_impl[s] = P
    for s in range(wl.B):
        for t in range(P * bs, int(wl.lens[s])):
            spec.reserve_slot(t_spec[s], t)
            n_impl[s] = impl.reserve_slot(t_impl[s], int(n_impl[s]), t)[1]
        assert t_impl[s, :n_impl[s]].tolist() == t_spec[s]
        assert t_spec[s] == wl.block_tables[s][wl.block_tables[s] >= 0].tolist()
    assert impl.refcount(t_spec[0][0]) == wl.B == spec.refcount[t_spec[0][0]]
    out = _run(wl)
    seqs = [0, 17, 63]
    assert_close(out[torch.as_tensor(seqs, device="cuda")], oracle_subset(wl, seqs), "prefix")

    # beams: a parent of fork_len tokens, 3 forks -> 4 beams sharing every block
    parent_spec, parent_impl = [], np.full(cap, -1, np.int32)
    npar = 0
    for t in range(fork_len):
        spec.reserve_slot(parent_spec, t)
        npar = impl.reserve_slot(parent_impl, npar, t)[1]
    # the parent's blocks came off the free list (poisoned): give them data
    pid = torch.as_tensor(parent_impl[:npar], device="cuda", dtype=torch.long)
    wl.k_pool[pid] = normal_fp16((npar, Hkv, bs, D), 44, "cuda")
    wl.v_pool[pid] = normal_fp16((npar, Hkv, bs, D), 45, "cuda")
    beams_spec = [parent_spec] + [list(parent_spec) for _ in range(3)]
    beams_impl = np.full((4, cap), -1, np.int32)
    for b in range(4):
        beams_impl[b, :npar] = parent_impl[:npar]
        if b:
            spec.fork(parent_spec)
            impl.fork(parent_impl[:npar])
    nbeam = np.full(4, npar, np.int32)
    lens4 = np.full(4, fork_len, np.int32)
    slots, pairs = impl.reserve_slots(beams_impl, nbeam, lens4)
    exp = [spec.reserve_slot(beams_spec[b], fork_len) for b in range(4)]
    assert slots.tolist() == [e[1] for e in exp]
    exp_pairs = [(e[2], e[3]) for e in exp if e[2] >= 0]
    assert [tuple(p) for p in pairs.tolist()] == exp_pairs
    assert len(exp_pairs) == (0 if fork_len % bs == 0 else 3)
    kn = normal_fp16((4, Hkv, D), 41, "cuda")
    vn = normal_fp16((4, Hkv, D), 42, "cuda")
    Kh, Vh = wl.k_pool.cpu().numpy(), wl.v_pool.cpu().numpy()
    if exp_pairs:
        Kh, Vh = oracle.copy_blocks(Kh, Vh, np.array(exp_pairs, np.int32))
        pkv.paged_kv_copy_blocks(wl.k_pool, wl.v_pool, torch.as_tensor(pairs, device="cuda"))
    Kh, Vh = oracle.append(Kh, Vh, kn.cpu().numpy(), vn.cpu().numpy(), np.array([e[1] for e in exp]))
    pkv.paged_kv_append(kn, vn, torch.as_tensor(slots, device="cuda"), wl.k_pool, wl.v_pool)
    assert pkv.device_error() == 0
    assert np.array_equal(_u16(wl.k_pool), Kh.view(np.uint16))
    assert np.array_equal(_u16(wl.v_pool), Vh.view(np.uint16))
    qb = normal_fp16((4, 1, wl.spec.Hq, D), 43, "cuda")
    L4 = lens4 + 1
    outb = pkv.paged_decode_attention(qb, wl.k_pool, wl.v_pool, torch.as_tensor(beams_impl, device="cuda"),
                                      torch.as_tensor(L4, device="cuda"), wl.scale)
    tb = np.full((4, cap), -1, np.int32)
    for b in range(4):
        tb[b, :len(beams_spec[b])] = beams_spec[b]
    ref = oracle.paged_attention(qb.cpu().numpy(), Kh, Vh, tb, L4, scale=wl.scale)
    assert_close(outb, ref, f"beams forked at {fork_len}")
