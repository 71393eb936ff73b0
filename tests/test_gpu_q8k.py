"""GPU parity of the quantised K pool: int8 codes with per-channel scales, fp16
V.  Calibration and the quantising append are bit-exact against the oracle;
attention over the codes is within the attention tolerance of exact fp64
attention over the dequantised keys.  Oracle inputs are made by the oracle
(codes quantised on the host), never taken from the device."""
import numpy as np
import pytest
import torch

import oracle
from paged_helpers import assert_close
from workloads import make_workload, normal_fp16

import paged_kv_cache_371_b200 as pkv
from paged_kv_cache_371_b200 import _abi

pytestmark = pytest.mark.gpu


def _calibration(Hkv, D, seed):
    return normal_fp16((2048, Hkv, D), seed, "cpu").numpy()


def _tokens_of_pool(pool):
    """[nb][Hkv][bs][D] -> [nb*bs][Hkv][D] (slot order), a view change only."""
    nb, Hkv, bs, D = pool.shape
    return pool.permute(0, 2, 1, 3).reshape(nb * bs, Hkv, D).contiguous()


def _quantise_on_device(wl, scales_np):
    nb, Hkv, bs, D = wl.k_pool.shape
    sc = torch.as_tensor(scales_np, device="cuda")
    kq = torch.zeros((nb, Hkv, bs, D), dtype=torch.int8, device="cuda")
    vq = torch.zeros_like(wl.v_pool)
    slots = torch.arange(nb * bs, dtype=torch.int64, device="cuda")
    pkv.paged_kv_append_q8k(_tokens_of_pool(wl.k_pool), _tokens_of_pool(wl.v_pool), slots, sc, kq, vq)
    return kq, vq, sc


def _oracle_subset_q8k(wl, kq_dev, scales, seqs, q, q_len):
    """Blocks of `seqs` quantised by the oracle on the host; the device codes of
    those blocks must equal them; exact attention over the oracle's codes."""
    tables = wl.block_tables[seqs]
    lens = wl.lens[seqs].astype(np.int32)
    ids = np.unique(tables[tables >= 0])
    idx = torch.as_tensor(ids, device="cuda", dtype=torch.long)
    K = wl.k_pool[idx].cpu().numpy()
    V = wl.v_pool[idx].cpu().numpy()
    n, Hkv, bs, D = K.shape
    toks = K.transpose(0, 2, 1, 3).reshape(n * bs, Hkv, D).copy()
    vt = V.transpose(0, 2, 1, 3).reshape(n * bs, Hkv, D).copy()
    K8, V2 = oracle.append_q8k(np.zeros((n, Hkv, bs, D), np.int8), np.zeros_like(V), toks, vt,
                               np.arange(n * bs, dtype=np.int64), scales)
    assert np.array_equal(kq_dev[idx].cpu().numpy(), K8), "device codes differ from the oracle's"
    assert np.array_equal(V2.view(np.uint16), V.view(np.uint16))
    t2 = np.where(tables >= 0, np.searchsorted(ids, np.maximum(tables, 0)), -1).astype(np.int32)
    qq = q[torch.as_tensor(seqs, device=q.device)].cpu().numpy()
    return oracle.paged_attention_q8k(qq, K8, scales, V, t2, lens, scale=wl.scale, q_len=q_len)


def test_calibration_scales_bit_exact():
    for Hkv, D, seed in ((8, 128, 3), (2, 64, 4)):
        k = normal_fp16((3000, Hkv, D), seed, "cpu")
        k[:, 0, 5] = 0
        k[17, 1, 3] = -40.0
        got = pkv.paged_kv_k_scales(k.cuda()).cpu().numpy()
        ref = oracle.k_scales(k.numpy())
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("bs,Hkv,D", [(16, 8, 128), (8, 4, 64)])
def test_append_q8k_bit_exact(bs, Hkv, D):
    rng = np.random.Generator(np.random.PCG64(bs + D))
    nb, T = 40, 300
    scales = oracle.k_scales(_calibration(Hkv, D, 9)) * np.float32(0.5)  # some codes clamp
    scales[1, 7] = np.float32(0.25)                                      # exact half steps below
    kn = normal_fp16((T, Hkv, D), 10, "cpu").numpy()
    kn[:8, 1, 7] = np.array([0.125, 0.375, -0.125, -0.375, 0.625, 31.875, -32.125, 40], np.float16)
    vn = normal_fp16((T, Hkv, D), 11, "cpu").numpy()
    slots = rng.permutation(nb * bs)[:T].astype(np.int64)
    slots[::37] = -1
    k0 = rng.integers(-128, 128, size=(nb, Hkv, bs, D)).astype(np.int8)
    v0 = normal_fp16((nb, Hkv, bs, D), 12, "cpu").numpy()
    kq, vq = torch.as_tensor(k0).cuda(), torch.as_tensor(v0).cuda()
    pkv.paged_kv_append_q8k(torch.as_tensor(kn).cuda(), torch.as_tensor(vn).cuda(),
                            torch.as_tensor(slots).cuda(), torch.as_tensor(scales).cuda(), kq, vq)
    K8, V2 = oracle.append_q8k(k0, v0, kn, vn, slots, scales)
    assert np.array_equal(kq.cpu().numpy(), K8)
    assert np.array_equal(vq.cpu().numpy().view(np.uint16), V2.view(np.uint16))
    assert pkv.device_error() == 0


def test_append_q8k_flags_bad_scale():
    kq = torch.zeros((4, 1, 16, 64), dtype=torch.int8, device="cuda")
    vq = torch.zeros((4, 1, 16, 64), dtype=torch.float16, device="cuda")
    sc = torch.ones((1, 64), dtype=torch.float32, device="cuda")
    sc[0, 3] = 0.0
    kn = torch.ones((1, 1, 64), dtype=torch.float16, device="cuda")
    pkv.device_error(reset=True)
    pkv.paged_kv_append_q8k(kn, kn, torch.tensor([5], dtype=torch.int64, device="cuda"), sc, kq, vq)
    assert pkv.device_error(reset=True) & _abi.KV_DEV_BAD_SCALE
    assert kq[0, 0, 5, 3].item() == 0 and kq[0, 0, 5, 2].item() == 1


@pytest.mark.parametrize("name,B,seqs", [
    ("llama7b_mha", 12, [0, 5, 11]),              # MHA (FMA path), outlier K channels
    ("llama70b_gqa", 24, [0, 7, 23]),             # GQA 8 rows (tensor-core path)
    ("llama70b_gqa_bs8", 16, [2, 9]),             # GQA, 8-token blocks
    ("long_verify", 2, [1]),                      # 5-token window x 4 heads (two m-tiles), 32K tokens
    ("long_decode", 2, [0]),                      # one long sequence: context splits + merge
])
def test_attention_q8k_matches_oracle(name, B, seqs):
    wl = make_workload(name, "cuda", B=B)
    nb, Hkv, bs, D = wl.k_pool.shape
    if D != 128:
        pytest.skip("int8 K pools are served at head_dim 128")
    q_len = wl.q.shape[1]
    scales = oracle.k_scales(_calibration(Hkv, D, 21))
    kq, vq, sc = _quantise_on_device(wl, scales)
    bt, cl = torch.as_tensor(wl.block_tables, device="cuda"), torch.as_tensor(wl.lens, device="cuda")
    out = pkv.paged_attention_q8k(wl.q, kq, sc, vq, bt, cl, wl.scale, q_len=q_len)
    torch.cuda.synchronize()
    assert pkv.device_error() == 0
    ref = _oracle_subset_q8k(wl, kq, scales, np.asarray(seqs), wl.q, q_len)
    assert_close(out[torch.as_tensor(seqs, device="cuda")], ref, f"q8k {name}")


def test_attention_q8k_edge_cases():
    """Empty and one-token contexts, a context ending mid-block, exact
    power-of-two scales (dequantised keys are fp16 values: the int8 path must
    then agree with the fp16 path within rounding of the scaled q)."""
    Hq, Hkv, D, bs = 8, 8, 128, 16
    lens = np.array([0, 1, 17, 300], np.int32)
    nb = 32
    rng = np.random.Generator(np.random.PCG64(5))
    codes = rng.integers(-127, 128, size=(nb, Hkv, bs, D)).astype(np.int8)
    scales = np.ldexp(1.0, -rng.integers(5, 8, size=(Hkv, D))).astype(np.float32)
    V = normal_fp16((nb, Hkv, bs, D), 6, "cpu").numpy()
    tables = np.full((4, 20), -1, np.int32)
    perm = rng.permutation(nb).astype(np.int32)
    off = 0
    for s, L in enumerate(lens):
        n = max(1, -(-int(L) // bs))
        tables[s, :n] = perm[off:off + n]
        off += n
    q = normal_fp16((4, 1, Hq, D), 7, "cuda")
    dev = lambda a: torch.as_tensor(a).cuda()
    out = pkv.paged_attention_q8k(q, dev(codes), dev(scales), dev(V), dev(tables), dev(lens), D ** -0.5)
    torch.cuda.synchronize()
    ref = oracle.paged_attention_q8k(q.cpu().numpy(), codes, scales, V, tables, lens, scale=D ** -0.5)
    assert_close(out, ref, "q8k edge cases")
    assert torch.count_nonzero(out[0]) == 0
    # one token: the output is that token's V
    t0 = tables[1, 0]
    assert torch.equal(out[1, 0].cpu(), torch.as_tensor(V[t0, :, 0, :]).repeat_interleave(Hq // Hkv, 0))
    kdq = (codes.astype(np.float64) * scales[None, :, None, :]).astype(np.float16)
    out16 = pkv.paged_decode_attention(q, dev(kdq), dev(V), dev(tables), dev(lens), D ** -0.5)
    torch.cuda.synchronize()
    assert_close(out, out16.cpu().double().numpy(), "int8 vs fp16 keys")


def test_copy_blocks_q8k_is_a_block_copy():
    nb, Hkv, bs, D = 12, 4, 16, 128
    rng = np.random.Generator(np.random.PCG64(3))
    k0 = rng.integers(-128, 128, size=(nb, Hkv, bs, D)).astype(np.int8)
    v0 = normal_fp16((nb, Hkv, bs, D), 4, "cpu").numpy()
    kq, vq = torch.as_tensor(k0).cuda(), torch.as_tensor(v0).cuda()
    pairs = np.array([[1, 7], [3, 0], [11, 5]], np.int32)
    pkv.paged_kv_copy_blocks_q8k(kq, vq, torch.as_tensor(pairs).cuda())
    torch.cuda.synchronize()
    k_ref = k0.copy()
    for src, dst in pairs:
        k_ref[dst] = k0[src]
    _, v_ref = oracle.copy_blocks(v0, v0, pairs)
    assert np.array_equal(kq.cpu().numpy(), k_ref)
    assert np.array_equal(vq.cpu().numpy().view(np.uint16), v_ref.view(np.uint16))



def _pool_scales(wl):
    """Channel scales from every token of the pool (unused rows, which hold
    NaN, count as zeros), computed by the oracle on the host."""
    K = np.nan_to_num(wl.k_pool.cpu().numpy())
    nb, Hkv, bs, D = K.shape
    return oracle.k_scales(K.transpose(0, 2, 1, 3).reshape(nb * bs, Hkv, D))


@pytest.mark.parametrize("name", ["llama7b_mha", "llama70b_gqa", "llama70b_gqa_bs8", "long_verify"])
def test_attention_q8k_full_size_every_sequence(name):
    """The int8-K forms of the benchmark's workloads at full size (scales from
    the whole pool, as the benchmark sets them), launched as the benchmark
    launches them: device codes bit-exact against the oracle's, and every
    output element of every sequence within tolerance."""
    wl = make_workload(name, "cuda")
    q_len = wl.q.shape[1]
    scales = _pool_scales(wl)
    kq, vq, sc = _quantise_on_device(wl, scales)
    bt, cl = torch.as_tensor(wl.block_tables, device="cuda"), torch.as_tensor(wl.lens, device="cuda")
    out = pkv.paged_attention_q8k(wl.q, kq, sc, vq, bt, cl, wl.scale, q_len=q_len)
    torch.cuda.synchronize()
    assert pkv.device_error() == 0
    ref = _oracle_subset_q8k(wl, kq, scales, np.arange(wl.B), wl.q, q_len)
    assert_close(out, ref, f"q8k {name} full size")


@pytest.mark.parametrize("Hq,Hkv,bs,q_len", [(8, 8, 16, 1), (64, 8, 16, 1), (64, 8, 8, 1),
                                             (32, 8, 16, 5)])
@pytest.mark.parametrize("grid,min_split", [(0, 0), (300, 1), (7, 1)])
def test_attention_q8k_planted_late_maxima(Hq, Hkv, bs, q_len, grid, min_split):
    """Dominant keys planted after the first stage (see planted.py) over an
    int8 K pool: FMA, one-tile and two-tile tensor-core consumers, with and
    without forced context splits."""
    from planted import plant
    lens = np.array([1500, 700, 333], np.int32)
    wl = make_workload("llama70b_gqa", "cuda", lens=lens, bs=bs, q_len=q_len, Hq=Hq, Hkv=Hkv,
                       D=128, seed=29 + Hq + bs + q_len)
    plan = {s: [(70, 40.0), (300, 80.0), (int(L) - 10, 120.0), (int(L) - 1, 160.0)]
            for s, L in enumerate(lens)}
    plant(wl, plan, seed=3 + Hq)
    scales = _pool_scales(wl)
    kq, vq, sc = _quantise_on_device(wl, scales)
    bt, cl = torch.as_tensor(wl.block_tables, device="cuda"), torch.as_tensor(wl.lens, device="cuda")
    out = pkv.paged_attention_q8k(wl.q, kq, sc, vq, bt, cl, wl.scale, q_len=q_len, grid_ctas=grid,
                                  min_split_blocks=min_split)
    torch.cuda.synchronize()
    assert pkv.device_error() == 0
    ref = _oracle_subset_q8k(wl, kq, scales, np.arange(wl.B), wl.q, q_len)
    assert_close(out, ref, f"q8k planted Hq{Hq} bs{bs} q{q_len}")
