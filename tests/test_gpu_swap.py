"""GPU: block swap between the pools and pinned host memory, and a prefix
found by content feeding decode attention (through the C ABI)."""
import time

import numpy as np
import pytest
import torch

import oracle
from oracle.block_spec import BlockPoolSpec, PrefixCacheSpec
from paged_helpers import assert_close
from workloads import normal_fp16

import paged_kv_cache_371_b200 as pkv
from paged_kv_cache_371_b200 import _abi

pytestmark = pytest.mark.gpu


def _pools(nb, Hkv, bs, D, seed):
    k = normal_fp16((nb, Hkv, bs, D), seed, "cuda")
    v = normal_fp16((nb, Hkv, bs, D), seed + 1, "cuda")
    return k, v


@pytest.mark.parametrize("bs,Hkv,D,n", [(16, 8, 128, 37), (8, 4, 64, 5), (16, 32, 128, 256)])
def test_swap_out_in_round_trip_is_a_block_copy(bs, Hkv, D, n):
    nb = 2 * n + 11
    k, v = _pools(nb, Hkv, bs, D, 71 + bs)
    rng = np.random.Generator(np.random.PCG64(n))
    perm = rng.permutation(nb)
    out_ids, in_ids = perm[:n].astype(np.int32), perm[n:2 * n].astype(np.int32)
    k0, v0 = k.cpu().numpy(), v.cpu().numpy()
    nbytes = pkv.swap_staging_bytes(k, n)
    staging = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    host = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    pkv.paged_kv_swap_out(k, v, torch.as_tensor(out_ids, device="cuda"), staging, host)
    torch.cuda.synchronize()
    # host = [K of out_ids ; V of out_ids], bit-exact
    h = host.view(torch.float16).view(2, n, Hkv, bs, D).numpy()
    assert np.array_equal(h[0].view(np.uint16), k0[out_ids].view(np.uint16))
    assert np.array_equal(h[1].view(np.uint16), v0[out_ids].view(np.uint16))
    staging.zero_()  # the swap-in must come from the host copy
    pkv.paged_kv_swap_in(k, v, torch.as_tensor(in_ids, device="cuda"), staging, host)
    torch.cuda.synchronize()
    kr, vr = oracle.copy_blocks(k0, v0, np.stack([out_ids, in_ids], 1))
    assert np.array_equal(k.cpu().numpy().view(np.uint16), kr.view(np.uint16))
    assert np.array_equal(v.cpu().numpy().view(np.uint16), vr.view(np.uint16))
    assert pkv.device_error() == 0


def test_swapped_sequence_attends_identically():
    """A sequence swapped out and back into other blocks gives the same
    attention output, bit for bit (same logical order), and matches the
    oracle."""
    bs, Hkv, Hq, D, L = 16, 8, 64, 128, 1000
    nblk = -(-L // bs)
    nb = 3 * nblk
    k, v = _pools(nb, Hkv, bs, D, 5)
    table = np.arange(nblk, dtype=np.int32)[None]
    q = normal_fp16((1, 1, Hq, D), 6, "cuda")
    lens = torch.tensor([L], dtype=torch.int32, device="cuda")
    scale = D ** -0.5
    out1 = pkv.paged_decode_attention(q, k, v, torch.as_tensor(table, device="cuda"), lens, scale)
    nbytes = pkv.swap_staging_bytes(k, nblk)
    staging = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    host = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    pkv.paged_kv_swap_out(k, v, torch.as_tensor(table[0], device="cuda"), staging, host)
    k[:nblk].fill_(float("nan"))   # the old blocks are reused by someone else
    v[:nblk].fill_(float("nan"))
    new = (np.arange(nblk, dtype=np.int32) + 2 * nblk)[::-1].copy()
    pkv.paged_kv_swap_in(k, v, torch.as_tensor(new, device="cuda"), staging, host)
    out2 = pkv.paged_decode_attention(q, k, v, torch.as_tensor(new[None], device="cuda"), lens, scale)
    torch.cuda.synchronize()
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    ref = oracle.paged_attention(q.cpu().numpy(), k.cpu().numpy(), v.cpu().numpy(), new[None],
                                 np.array([L], np.int32), scale=scale)
    assert_close(out2, ref, "after swap-in")


def test_swap_bad_id_is_flagged_and_skipped():
    k, v = _pools(8, 2, 16, 64, 9)
    k0 = k.clone()
    staging = torch.zeros(pkv.swap_staging_bytes(k, 2), dtype=torch.uint8, device="cuda")
    pkv.device_error(reset=True)
    pkv.paged_kv_swap_in(k, v, torch.tensor([3, 99], dtype=torch.int32, device="cuda"), staging)
    torch.cuda.synchronize()
    assert pkv.device_error(reset=True) & _abi.KV_DEV_BAD_BLOCK
    assert torch.equal(k[3], torch.zeros_like(k[3]))     # the valid row was written
    mask = torch.ones(8, dtype=torch.bool)
    mask[3] = False
    assert torch.equal(k[mask.cuda()], k0[mask.cuda()])   # nothing else changed


def test_swap_bandwidth_is_reported():
    """Device -> pinned host -> device for 1024 blocks of a 70B-shaped pool
    (64 MiB each way); prints the achieved rates."""
    bs, Hkv, D, n = 16, 8, 128, 1024
    k, v = _pools(2 * n, Hkv, bs, D, 13)
    ids = torch.arange(n, dtype=torch.int32, device="cuda")
    nbytes = pkv.swap_staging_bytes(k, n)
    staging = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    host = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    for _ in range(2):
        pkv.paged_kv_swap_out(k, v, ids, staging, host)
        pkv.paged_kv_swap_in(k, v, ids + n, staging, host)
    torch.cuda.synchronize()
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    e[0].record()
    pkv.paged_kv_swap_out(k, v, ids, staging, host)
    e[1].record()
    pkv.paged_kv_swap_in(k, v, ids + n, staging, host)
    e[2].record()
    torch.cuda.synchronize()
    t_out, t_in = e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2])
    print(f"\nswap {nbytes / 2**20:.0f} MiB: out {nbytes / t_out / 1e6:.1f} GB/s, "
          f"in {nbytes / t_in / 1e6:.1f} GB/s")
    assert torch.equal(k[:n], k[n:]) and torch.equal(v[:n], v[n:])


def test_prefix_found_by_content_feeds_decode():
    """Request A computes a 3-block system prompt + its own question and
    registers its blocks; request B with the same system prompt matches them
    by content, appends only its own tokens, and its decode attention over
    the shared table equals the oracle over a private copy."""
    bs, Hkv, Hq, D = 16, 8, 32, 128
    nb = 64
    pool = pkv.KVPool(nb, bs, Hkv, D)
    spool = BlockPoolSpec(nb, bs)
    scache = PrefixCacheSpec(spool)
    k = torch.zeros((nb, Hkv, bs, D), dtype=torch.float16, device="cuda")
    v = torch.zeros_like(k)
    system = list(range(500, 500 + 3 * bs))
    tok_a = system + list(range(900, 920))
    tok_b = system + list(range(700, 737))

    def admit(tokens, seed):
        table = pool.prefix_match(tokens)
        st, stab = scache.match(tokens)
        assert table == stab
        n_cached = len(table) * bs
        need = -(-len(tokens) // bs) - len(table)
        ids = pool.alloc(need)
        assert spool.alloc(need)[1] == ids
        table = table + ids
        T = len(tokens) - n_cached   # only the uncached tokens are computed and appended
        kn = normal_fp16((T, Hkv, D), seed, "cuda")
        vn = normal_fp16((T, Hkv, D), seed + 1, "cuda")
        slots = [table[t // bs] * bs + t % bs for t in range(n_cached, len(tokens))]
        pkv.paged_kv_append(kn, vn, torch.as_tensor(slots, dtype=torch.int64, device="cuda"), k, v)
        assert pool.prefix_register(tokens, table) == scache.register(tokens, table)[1]
        return table, n_cached

    ta, ca = admit(tok_a, 11)
    tb, cb = admit(tok_b, 21)
    assert ca == 0 and cb == 3 * bs and tb[:3] == ta[:3]
    assert [pool.refcount(b) for b in ta[:3]] == [3, 3, 3]
    cap = max(len(ta), len(tb))
    tables = np.full((2, cap), -1, np.int32)
    tables[0, :len(ta)] = ta
    tables[1, :len(tb)] = tb
    lens = np.array([len(tok_a), len(tok_b)], np.int32)
    q = normal_fp16((2, 1, Hq, D), 31, "cuda")
    out = pkv.paged_decode_attention(q, k, v, torch.as_tensor(tables, device="cuda"),
                                     torch.as_tensor(lens, device="cuda"), D ** -0.5)
    torch.cuda.synchronize()
    # oracle over private copies: each sequence's blocks copied into a fresh
    # contiguous layout (shared blocks duplicated)
    K, V = k.cpu().numpy(), v.cpu().numpy()
    ref = []
    for s, t in enumerate((ta, tb)):
        ref.append(oracle.paged_attention(q[s:s + 1].cpu().numpy(), K[t], V[t],
                                          np.arange(len(t), dtype=np.int32)[None], lens[s:s + 1],
                                          scale=D ** -0.5))
    assert_close(out, np.concatenate(ref), "shared system prompt")
