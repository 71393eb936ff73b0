"""The two compute paths for several query rows per KV head (head_dim 128),
each against the fp64 oracle on the same seeded inputs (needs a B200):

  consumer=1  warp-level tensor-core MMAs, accumulators in registers
  consumer=2  tcgen05 MMAs, accumulators in tensor memory (each TMEM lane one
              query row and a slice of the stage's tokens; the slices of a row
              merged at the end of every segment)

Oracle-sized problems over several stages and ragged tails, forced context
splits, planted late maxima (the lazy rescale of O in tensor memory), the
edge cases (empty context, one token, rows that see nothing), int8 keys, the
full-size verify and GQA workloads, and bit-reproducibility.
"""
import numpy as np
import pytest
import torch

from paged_helpers import assert_close, device_inputs, oracle_subset
from workloads import make_workload, normal_fp16

pytestmark = pytest.mark.gpu

pkv = pytest.importorskip("paged_kv_cache_371_b200")


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    pkv.device_error(reset=True)
    yield
    torch.cuda.synchronize()


def _run(wl, q_len, **kw):
    bt, cl = device_inputs(wl)
    out = pkv.paged_attention(wl.q, wl.k_pool, wl.v_pool, bt, cl, wl.scale, q_len=q_len, **kw)
    torch.cuda.synchronize()
    assert pkv.device_error() == 0
    return out


SHAPES = [
    (64, 8, 16, 1),    # GQA 8: 8 rows (tcgen05 rows padded to 8)
    (64, 8, 8, 1),     # the same over 8-token blocks
    (24, 2, 16, 1),    # 12 rows (padded to 16)
    (32, 8, 8, 5),     # verify window 5 x 4 heads: 20 rows (padded to 32)
    (16, 2, 16, 4),    # 32 rows, no padding
    (32, 1, 16, 1),    # MQA: 32 rows
    (4, 4, 16, 3),     # one head per KV head, verify window 3: 3 rows
]


@pytest.mark.parametrize("Hq,Hkv,bs,q_len", SHAPES)
@pytest.mark.parametrize("grid,min_split", [(0, 0), (300, 1), (7, 1)])
@pytest.mark.parametrize("consumer", [1, 2])
def test_consumers_forced_splits(Hq, Hkv, bs, q_len, grid, min_split, consumer):
    rng = np.random.Generator(np.random.PCG64(Hq * 71 + bs + q_len))
    lens = np.array([1, bs, 3 * bs + 1, 200, 411, 1000], dtype=np.int32)
    lens = np.maximum(lens, q_len)
    wl = make_workload("llama70b_gqa", "cuda", lens=lens, bs=bs, q_len=q_len, Hq=Hq, Hkv=Hkv, D=128,
                       seed=int(rng.integers(1 << 30)))
    out = _run(wl, q_len, grid_ctas=grid, min_split_blocks=min_split, consumer=consumer)
    ref = oracle_subset(wl, list(range(wl.B)), q_len)
    assert_close(out, ref, f"consumer {consumer} Hq{Hq} Hkv{Hkv} bs{bs} q{q_len} grid{grid}")


@pytest.mark.parametrize("Hq,Hkv,bs,q_len", [(64, 8, 16, 1), (64, 8, 8, 1), (32, 8, 16, 5),
                                             (16, 2, 16, 4)])
@pytest.mark.parametrize("grid,min_split", [(0, 0), (300, 1), (7, 1)])
def test_tcgen05_planted_late_maxima(Hq, Hkv, bs, q_len, grid, min_split):
    """Aligned keys planted after the first stage and near the end, each
    dominating all before it: every lane's running maximum jumps past the
    lazy-rescale threshold, so O is rescaled in tensor memory mid-segment,
    and the partial rows of a split carry the jump into the merge."""
    from planted import plant
    lens = np.array([1500, 700, 333], np.int32)
    wl = make_workload("llama70b_gqa", "cuda", lens=lens, bs=bs, q_len=q_len, Hq=Hq, Hkv=Hkv, D=128,
                       seed=41 + Hq + bs + q_len)
    plan = {s: [(70, 40.0), (300, 80.0), (int(L) - 10, 120.0), (int(L) - 1, 160.0)]
            for s, L in enumerate(lens)}
    plant(wl, plan, seed=7 + Hq + q_len)
    out = _run(wl, q_len, grid_ctas=grid, min_split_blocks=min_split, consumer=2)
    ref = oracle_subset(wl, list(range(wl.B)), q_len)
    assert_close(out, ref, f"tcgen05 planted Hq{Hq} bs{bs} q{q_len} grid{grid}")


def test_tcgen05_ramped_keys():
    """Key norms growing along the context: the maximum keeps growing, many
    rescales per segment."""
    from planted import ramp
    lens = np.array([2000, 900], np.int32)
    wl = make_workload("llama70b_gqa", "cuda", lens=lens, q_len=5, Hq=32, Hkv=8, D=128, seed=5)
    ramp(wl, 150.0)
    out = _run(wl, 5, consumer=2, grid_ctas=9, min_split_blocks=1)
    assert_close(out, oracle_subset(wl, [0, 1], 5), "tcgen05 ramped keys")


def test_tcgen05_edge_cases():
    """Empty context (zeros), one token (exactly V), block multiples, a
    verify window longer than the context (rows that see nothing: zeros)."""
    lens = np.array([0, 1, 16, 17, 32, 2], dtype=np.int32)
    wl = make_workload("llama70b_gqa", "cuda", lens=lens, q_len=1, seed=78, Hq=8, Hkv=2, D=128)
    out = _run(wl, 1, grid_ctas=5, min_split_blocks=1, consumer=2)
    assert_close(out, oracle_subset(wl, list(range(len(lens)))), "tcgen05 edge decode")
    assert not out[0].any()
    v0 = wl.v_pool[int(wl.block_tables[1, 0]), :, 0, :]
    assert torch.equal(out[1, 0].view(torch.int16), v0.repeat_interleave(4, dim=0).view(torch.int16))
    wl.q = normal_fp16((len(lens), 3, 8, 128), 9, "cuda")
    out3 = _run(wl, 3, grid_ctas=3, consumer=2)
    assert_close(out3, oracle_subset(wl, list(range(len(lens))), q_len=3), "tcgen05 edge verify")
    assert not out3[0].any()


@pytest.mark.parametrize("name", ["long_verify", "llama70b_gqa", "llama70b_gqa_bs8"])
def test_tcgen05_full_size_every_sequence(name):
    """Full-size workloads on the tcgen05 path, launched as the benchmark
    launches them: every output of every sequence."""
    wl = make_workload(name, "cuda")
    q_len = wl.spec.q_len
    out = _run(wl, q_len, consumer=2)
    assert_close(out, oracle_subset(wl, list(range(wl.B)), q_len), f"tcgen05 {name}")


def test_tcgen05_bit_reproducible():
    """The slices of a row are merged in a fixed order: same launch, same bits."""
    wl = make_workload("long_verify", "cuda", B=2, max_len=5000)
    a = _run(wl, 5, consumer=2).clone()
    b = _run(wl, 5, consumer=2).clone()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("Hq,Hkv,bs,q_len", [(64, 8, 16, 1), (64, 8, 8, 1), (32, 8, 16, 5)])
@pytest.mark.parametrize("consumer", [1, 2])
def test_q8k_consumers(Hq, Hkv, bs, q_len, consumer):
    """int8 keys on both paths (the tcgen05 path widens the codes to fp16 in
    shared memory), planted late maxima, forced splits."""
    from planted import plant
    from test_gpu_q8k import _oracle_subset_q8k, _pool_scales, _quantise_on_device
    lens = np.array([1500, 700, 333, 17], np.int32)
    wl = make_workload("llama70b_gqa", "cuda", lens=lens, bs=bs, q_len=q_len, Hq=Hq, Hkv=Hkv, D=128,
                       seed=53 + Hq + bs + q_len)
    plan = {s: [(70, 40.0), (300, 80.0), (int(L) - 1, 160.0)] for s, L in enumerate(lens[:3])}
    plant(wl, plan, seed=11 + Hq)
    scales = _pool_scales(wl)
    kq, vq, sc = _quantise_on_device(wl, scales)
    bt, cl = torch.as_tensor(wl.block_tables, device="cuda"), torch.as_tensor(wl.lens, device="cuda")
    ref = _oracle_subset_q8k(wl, kq, scales, np.arange(wl.B), wl.q, q_len)
    for grid, ms in ((0, 0), (300, 1), (7, 1)):
        out = pkv.paged_attention_q8k(wl.q, kq, sc, vq, bt, cl, wl.scale, q_len=q_len, grid_ctas=grid,
                                      min_split_blocks=ms, consumer=consumer)
        torch.cuda.synchronize()
        assert pkv.device_error() == 0
        assert_close(out, ref, f"q8k consumer {consumer} Hq{Hq} bs{bs} q{q_len} grid{grid}")


def test_bad_consumer_value_is_rejected():
    wl = make_workload("llama70b_gqa", "cuda", B=2, max_len=100, seed=3)
    with pytest.raises(Exception):
        _run(wl, 1, consumer=3)
