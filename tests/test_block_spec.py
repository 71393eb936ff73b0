"""The bookkeeping spec (oracle/block_spec.py) against the pages' figures and
against invariants that any correct refcounted pool keeps (CPU only)."""
import numpy as np
import pytest

from conftest import read_golden
from oracle.block_spec import (ERR_DOUBLE_FREE, ERR_INVALID, ERR_OOM, OK,
                               BlockPoolSpec)


def _order(first, n):
    rest = [i for i in range(n) if i not in first]
    return list(first) + rest


def _grow(pool, table, start, stop):
    """Append tokens start..stop-1 one by one; returns their slots and copies."""
    slots, copies = [], []
    for t in range(start, stop):
        st, slot, src, dst = pool.reserve_slot(table, t)
        assert st == OK
        slots.append(slot)
        if src >= 0:
            copies.append((src, dst))
    return slots, copies


def test_logical_to_physical_figure():
    _, kv = read_golden("block_table_figure.txt")
    d = dict(kv)
    bs = int(d["block_size"][0])
    table_ref = [int(x) for x in d["table"]]
    pool = BlockPoolSpec(16, bs, _order(table_ref, 16))
    table = []
    slots, copies = _grow(pool, table, 0, int(d["tokens"][0]))
    assert table == table_ref and not copies
    for b, rng in enumerate(d["logical_token_ranges"]):
        lo, hi = (int(x) for x in rng.split("-"))
        for t in range(lo, hi + 1):
            assert slots[t] // bs == table_ref[b] and slots[t] % bs == t - lo


def test_three_requests_figure():
    _, kv = read_golden("three_requests_figure.txt")
    bs = int(dict(kv)["block_size"][0])
    reqs = [[int(x) for x in v] for k, v in kv if k == "request"]
    flat = [i for r in reqs for i in r]
    pool = BlockPoolSpec(16, bs, _order(flat, 16))
    for r in reqs:
        table = []
        _grow(pool, table, 0, len(r) * bs)
        assert table == r
    assert pool.num_free() == 16 - len(flat)


def test_copy_on_write_figure():
    _, kv = read_golden("cow_figure.txt")
    d = dict(kv)
    bs = int(d["block_size"][0])
    shared = int(d["shared_block"][0])
    src, dst = (int(x) for x in d["copy"])
    pool = BlockPoolSpec(32, bs, _order([shared, dst], 32))
    parent = []
    _grow(pool, parent, 0, 10)                 # partial block: 10 of 16 tokens
    beam_a, beam_b = parent, list(parent)      # beam A continues the parent's table
    assert pool.fork(beam_b) == OK             # beam B shares every block
    assert beam_a == beam_b == [shared] and pool.refcount[shared] == 2
    st, slot_b, s, t = pool.reserve_slot(beam_b, 10)   # beam B writes first
    assert st == OK and (s, t) == (src, dst) and slot_b == dst * bs + 10
    st, slot_a, s, t = pool.reserve_slot(beam_a, 10)   # then beam A, in place
    assert st == OK and (s, t) == (-1, -1) and slot_a == shared * bs + 10
    assert beam_a == [int(x) for x in d["after_A"]]
    assert beam_b == [int(x) for x in d["after_B"]]
    assert pool.refcount[shared] == 1 and pool.refcount[dst] == 1


def test_prefix_sharing_figure():
    _, kv = read_golden("prefix_sharing_figure.txt")
    d = dict(kv)
    bs = int(d["block_size"][0])
    prefix = [int(x) for x in d["prefix"]]
    suffixes = [[int(x) for x in v] for k, v in kv if k == "suffix"]
    pool = BlockPoolSpec(32, bs, _order(prefix + [i for s in suffixes for i in s], 32))
    first = []
    _grow(pool, first, 0, len(prefix) * bs)
    tables = [first]
    for _ in suffixes[1:]:
        assert pool.fork(first) == OK
        tables.append(list(first))
    assert all(pool.refcount[b] == len(suffixes) for b in prefix)
    n0 = len(prefix) * bs
    for table, suf in zip(tables, suffixes):
        _, copies = _grow(pool, table, n0, n0 + len(suf) * bs)
        assert not copies
        assert table == prefix + suf


def test_alloc_all_or_nothing_and_lifo_reuse():
    pool = BlockPoolSpec(4, 16)
    st, ids = pool.alloc(3)
    assert st == OK and ids == [0, 1, 2]
    assert pool.alloc(2) == (ERR_OOM, []) and pool.num_free() == 1
    assert pool.free([1, 0]) == OK
    st, ids = pool.alloc(3)
    assert ids == [0, 1, 3]        # last freed first, then the untouched one


def test_double_free_and_bad_ids():
    pool = BlockPoolSpec(4, 8)
    _, ids = pool.alloc(2)
    assert pool.free([ids[0], ids[0]]) == ERR_DOUBLE_FREE
    assert pool.refcount[ids[0]] == 1          # nothing changed
    assert pool.free([7]) == ERR_INVALID
    assert pool.fork([3]) == ERR_INVALID       # block 3 is free
    assert pool.reserve_slot([ids[0]], 0)[0] == ERR_INVALID   # table/len mismatch


def test_random_ops_keep_invariants():
    rng = np.random.Generator(np.random.PCG64(7))
    pool = BlockPoolSpec(64, 8, rng.permutation(64))
    seqs = []  # (table, length)
    for _ in range(3000):
        op = rng.integers(0, 4)
        if op == 0 or not seqs:
            seqs.append(([], 0))
        elif op == 1:
            i = int(rng.integers(len(seqs)))
            table, n = seqs[i]
            st, slot, src, dst = pool.reserve_slot(table, n)
            if st == OK:
                seqs[i] = (table, n + 1)
                assert slot // 8 == table[-1] and slot % 8 == n % 8
            else:
                assert st == ERR_OOM
        elif op == 2:
            i = int(rng.integers(len(seqs)))
            table, n = seqs[i]
            assert pool.fork(table) == OK
            seqs.append((list(table), n))
        else:
            i = int(rng.integers(len(seqs)))
            table, n = seqs.pop(i)
            assert pool.free(table) == OK
        # conservation: refcount == number of table references; free <=> 0
        refs = np.zeros(64, dtype=int)
        for table, _ in seqs:
            for b in table:
                refs[b] += 1
        assert list(refs) == pool.refcount
        assert sorted(pool.free_stack) == [b for b in range(64) if refs[b] == 0]
