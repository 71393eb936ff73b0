"""C-ABI library: loads, exports every declared symbol, and its host
bookkeeping matches the Python spec bit for bit (CPU only, no device calls)."""
import os
import re

import numpy as np
import pytest

from conftest import ROOT
from oracle.block_spec import BlockPoolSpec, OK as SPEC_OK

import paged_kv_cache_371_b200 as pkv
from paged_kv_cache_371_b200 import _abi

HEADER = os.path.join(ROOT, "include", "paged_kv.h")


def declared_functions():
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^(?:const\s+)?\w+\**\s+\**(\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_expected_calls():
    names = declared_functions()
    for must in ("kv_pool_create", "block_alloc", "block_free", "block_fork",
                 "kv_seq_reserve_slot", "paged_kv_append", "paged_kv_copy_blocks",
                 "paged_decode_attention", "paged_verify_attention", "kv_device_error"):
        assert must in names


def test_library_exports_every_declared_symbol():
    L = pkv.lib()
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing
    assert set(declared_functions()) <= set(_abi.SIGNATURES)


def test_pool_bytes_matches_oracle_formula():
    import oracle
    for nb, bs, hkv, d, layers in [(1000, 16, 8, 128, 80), (16, 16, 4, 64, 1), (9216, 8, 32, 128, 2)]:
        per, tot = pkv.pool_bytes(nb, bs, hkv, d, layers)
        assert per == oracle.pool_bytes_per_layer(nb, bs, hkv, d, 2)
        assert tot == per * layers


def test_errors_are_reported_not_raised_natively():
    pool = pkv.KVPool(4, 16)
    ids = pool.alloc(4)
    with pytest.raises(pkv.KVError) as e:
        pool.alloc(1)
    assert e.value.code == _abi.KV_ERR_OOM
    pool.free(ids[:1])
    with pytest.raises(pkv.KVError) as e:
        pool.free(ids[:1])
    assert e.value.code == _abi.KV_ERR_DOUBLE_FREE
    with pytest.raises(pkv.KVError):
        pkv.KVPool(4, 12)  # block size must be 8 or 16
    with pytest.raises(pkv.KVError):
        pkv.KVPool(3, 16, order=[0, 0, 1])


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_block_manager_matches_spec(seed):
    """Random alloc / fork / append / free sequences: identical ids, tables,
    slots, copy pairs, refcounts and free counts."""
    rng = np.random.Generator(np.random.PCG64(seed))
    nb, bs, cap = 48, (8, 16, 16)[seed % 3], 64
    order = rng.permutation(nb)
    spec = BlockPoolSpec(nb, bs, order)
    impl = pkv.KVPool(nb, bs, order=order)
    seqs = []  # [spec_table(list), impl_table(np), n_blocks, length]
    for step in range(2500):
        op = int(rng.integers(0, 10))
        if op == 0 or not seqs:
            seqs.append([[], np.full(cap, -1, np.int32), 0, 0])
        elif op <= 6:
            i = int(rng.integers(len(seqs)))
            st_tab, im_tab, nblk, n = seqs[i]
            st, slot, src, dst = spec.reserve_slot(st_tab, n)
            if st == SPEC_OK:
                got = impl.reserve_slot(im_tab, nblk, n)
                assert got == (slot, len(st_tab), src, dst)
                seqs[i][2] = got[1]
                seqs[i][3] = n + 1
            else:
                with pytest.raises(pkv.KVError):
                    impl.reserve_slot(im_tab, nblk, n)
        elif op <= 7:
            i = int(rng.integers(len(seqs)))
            st_tab, im_tab, nblk, n = seqs[i]
            assert spec.fork(st_tab) == SPEC_OK
            impl.fork(im_tab[:nblk])
            seqs.append([list(st_tab), im_tab.copy(), nblk, n])
        else:
            i = int(rng.integers(len(seqs)))
            st_tab, im_tab, nblk, n = seqs.pop(i)
            assert spec.free(st_tab) == SPEC_OK
            impl.free(im_tab[:nblk])
        for st_tab, im_tab, nblk, _ in seqs:
            assert list(im_tab[:nblk]) == st_tab
        assert impl.num_free() == spec.num_free()
        if step % 97 == 0:
            assert [impl.refcount(b) for b in range(nb)] == spec.refcount


def test_batch_reserve_matches_sequential_spec():
    rng = np.random.Generator(np.random.PCG64(9))
    nb, bs, B, cap = 256, 16, 12, 40
    order = rng.permutation(nb)
    spec = BlockPoolSpec(nb, bs, order)
    impl = pkv.KVPool(nb, bs, order=order)
    lens = rng.integers(0, 200, size=B).astype(np.int32)
    tables = np.full((B, cap), -1, np.int32)
    nblk = np.zeros(B, np.int32)
    spec_tables = [[] for _ in range(B)]
    for s in range(B):  # build the sequences token by token
        for t in range(int(lens[s])):
            spec.reserve_slot(spec_tables[s], t)
            impl.reserve_slot(tables[s], int(nblk[s]), t)
            nblk[s] = len(spec_tables[s])
    # share some sequences' blocks to force copy-on-write in the batch
    for s in range(0, B, 3):
        spec.fork(spec_tables[s])
        impl.fork(tables[s, :nblk[s]])
    for step in range(5):
        slots, pairs = impl.reserve_slots(tables, nblk, lens)
        exp_slots, exp_pairs = [], []
        for s in range(B):
            st, slot, src, dst = spec.reserve_slot(spec_tables[s], int(lens[s]))
            assert st == SPEC_OK
            exp_slots.append(slot)
            if src >= 0:
                exp_pairs.append((src, dst))
        assert slots.tolist() == exp_slots
        assert [tuple(p) for p in pairs.tolist()] == exp_pairs
        for s in range(B):
            assert tables[s, :nblk[s]].tolist() == spec_tables[s]
        lens = lens + 1


def test_workspace_size_covers_the_head_pair_form():
    """The split partials are [grid][2][rows][head_dim] fp32 plus one log-sum
    per row and 16 bytes of metadata per CTA.  A shape the kernel may serve as
    pairs of KV heads (head_dim 128, one query, an even number of KV heads,
    groups of 1, 2, 4 or 8) is sized for two 8-row tiles, 16 rows, whatever
    its group size; others for their rows padded to 16 (1 for one row)."""
    grid = 148

    def expect(rp, D):
        lse = (grid * 2 * rp * 4 + 15) // 16 * 16
        return grid * 16 + lse + grid * 2 * rp * D * 4

    cases = [  # (Hq, Hkv, q_len, D, padded rows)
        (32, 32, 1, 128, 16),   # MHA, head_dim 128: pairs possible
        (32, 32, 1, 64, 1),     # MHA, head_dim 64: one row
        (31, 31, 1, 128, 1),    # odd KV heads: no pairs
        (32, 8, 1, 128, 16),    # GQA 4
        (64, 8, 1, 128, 16),    # GQA 8
        (32, 8, 5, 128, 32),    # 5-token verify window, 20 rows
        (32, 1, 1, 128, 32),    # MQA, 32 rows
        (16, 16, 3, 128, 16),   # MHA verify window of 3 rows
    ]
    for Hq, Hkv, q_len, D, rp in cases:
        assert pkv.workspace_size(Hq, Hkv, q_len, D, grid) == expect(rp, D), (Hq, Hkv, q_len, D)
