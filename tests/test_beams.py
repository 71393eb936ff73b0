"""Beam-search bookkeeping: the spec's reorder step pinned against the pages'
beam example and conservation laws, and the C++ step checked against the
spec bit for bit over many random beam-search steps (CPU only)."""
import numpy as np
import pytest

from oracle.block_spec import OK, ERR_INVALID, BlockPoolSpec, beam_reorder

import paged_kv_cache_371_b200 as pkv


def _grow(pool, table, n0, n1):
    for t in range(n0, n1):
        st, _, _, _ = pool.reserve_slot(table, t)
        assert st == OK


def _conserved(pool, tables):
    refs = np.zeros(pool.num_blocks, np.int64)
    for t in tables:
        for b in t:
            refs[b] += 1
    assert refs.tolist() == pool.refcount
    assert not (set(pool.free_stack) & {b for t in tables for b in t})
    assert len(pool.free_stack) + int((refs > 0).sum()) == pool.num_blocks


def test_four_beams_at_1024_tokens_share_every_block():
    """[T3] §2.3 (2): 4 beams of a 1024-token sequence share its blocks; the
    next token gives each beam one new block: 64 + 4 blocks instead of
    4 x 65 private ones."""
    pool = BlockPoolSpec(400, 16)
    parent = []
    _grow(pool, parent, 0, 1024)
    st, beams = beam_reorder(pool, [parent], [0, 0, 0, 0])
    assert st == OK and all(b == parent for b in beams)
    assert all(pool.refcount[b] == 4 for b in parent)
    copies = []
    for b in beams:
        st, slot, src, dst = pool.reserve_slot(b, 1024)
        copies.append(src)
    assert copies == [-1] * 4                    # 1024 = 64 x 16: no copy
    used = sum(1 for r in pool.refcount if r > 0)
    assert used == 64 + 4 and 4 * 65 == 260
    _conserved(pool, beams)


def test_partial_last_block_is_copied_for_all_but_one_writer():
    pool = BlockPoolSpec(64, 16)
    parent = []
    _grow(pool, parent, 0, 40)                   # last block 8/16 full
    st, beams = beam_reorder(pool, [parent], [0, 0, 0])
    pairs = []
    for b in beams:
        st, slot, src, dst = pool.reserve_slot(b, 40)
        if src >= 0:
            pairs.append((src, dst))
    assert len(pairs) == 2 and all(s == parent[-1] for s, _ in pairs)
    assert pool.refcount[parent[-1]] == 1        # the last writer keeps it
    _conserved(pool, beams)


def test_identity_reorder_changes_nothing():
    pool = BlockPoolSpec(32, 8)
    tables = []
    for n in (5, 17, 30):
        t = []
        _grow(pool, t, 0, n)
        tables.append(t)
    before = (list(pool.refcount), list(pool.free_stack))
    st, new = beam_reorder(pool, tables, [0, 1, 2])
    assert st == OK and new == tables
    assert (list(pool.refcount), list(pool.free_stack)) == before


def test_dropped_beams_free_their_private_blocks_in_order():
    pool = BlockPoolSpec(32, 4)
    a, b = [], []
    _grow(pool, a, 0, 8)
    _grow(pool, b, 0, 6)
    st, new = beam_reorder(pool, [a, b], [0, 0])
    assert st == OK and new == [a, a]
    assert pool.free_stack[-2:] == b            # b's blocks, in table order
    assert beam_reorder(pool, new, [5]) == (ERR_INVALID, [])
    _conserved(pool, new)


@pytest.mark.parametrize("seed,bs", [(1, 16), (2, 8)])
def test_cpp_beam_search_matches_spec(seed, bs):
    """S prompts x W beams for many steps: random survivors inside each
    prompt's beams, batched slot reservation with copy-on-write; identical
    tables, slots, copy pairs, refcounts and free counts; conservation."""
    rng = np.random.Generator(np.random.PCG64(seed))
    S, W, nb, cap = 6, 5, 600, 64
    order = rng.permutation(nb)
    spec = BlockPoolSpec(nb, bs, order)
    impl = pkv.KVPool(nb, bs, order=order)
    lens0 = rng.integers(1, 6 * bs, size=S)
    st_tabs = []
    im_tabs = np.full((S, cap), -1, np.int32)
    im_nb = np.zeros(S, np.int32)
    for s in range(S):
        t = []
        _grow(spec, t, 0, int(lens0[s]))
        st_tabs.append(t)
        for x in range(int(lens0[s])):
            im_nb[s] = impl.reserve_slot(im_tabs[s], int(im_nb[s]), x)[1]
        assert im_tabs[s, :im_nb[s]].tolist() == t
    # rows of the current beam tables: prompt groups of W beams each
    parents = np.repeat(np.arange(S), W).astype(np.int32)
    beam_len = lens0.astype(np.int32)       # length of every current row
    n_groups = S
    n_pairs = 0
    for step in range(40):
        st, st_tabs = beam_reorder(spec, st_tabs, parents.tolist())
        assert st == OK
        im_tabs, im_nb = impl.beam_reorder(im_tabs, im_nb, parents)
        for i, t in enumerate(st_tabs):
            assert im_tabs[i, :im_nb[i]].tolist() == t
        lens = beam_len[parents].astype(np.int32)
        exp = [spec.reserve_slot(st_tabs[i], int(lens[i])) for i in range(len(st_tabs))]
        assert all(e[0] == OK for e in exp)
        slots, pairs = impl.reserve_slots(im_tabs, im_nb, lens)
        assert slots.tolist() == [e[1] for e in exp]
        assert [tuple(p) for p in pairs.tolist()] == [(e[2], e[3]) for e in exp if e[2] >= 0]
        n_pairs += len(pairs)
        beam_len = lens + 1
        assert impl.num_free() == spec.num_free()
        assert [impl.refcount(b) for b in range(nb)] == spec.refcount
        _conserved(spec, st_tabs)
        # survivors: each prompt keeps W beams drawn from its own W beams;
        # at step 25 every other prompt finishes
        groups = range(n_groups) if step != 25 else range(0, n_groups, 2)
        parents = np.concatenate([g * W + rng.integers(0, W, size=W) for g in groups]).astype(np.int32)
        n_groups = len(groups)
    assert n_pairs > 20
