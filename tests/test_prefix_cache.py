"""Prefix cache: the Python spec pinned against the pages' figure and the
properties a prefix cache must have, then the C++ cache checked against the
spec bit for bit (CPU only)."""
import numpy as np
import pytest

from conftest import read_golden
from oracle.block_spec import OK, BlockPoolSpec, PrefixCacheSpec, beam_reorder

import paged_kv_cache_371_b200 as pkv


def _order(first, n):
    rest = [i for i in range(n) if i not in first]
    return list(first) + rest


def _request(pool, cache, tokens):
    """A request arrives: match its cached prefix, allocate the rest."""
    bs = pool.block_size
    st, table = cache.match(tokens)
    assert st == OK
    need = -(-len(tokens) // bs) - len(table)
    st, ids = pool.alloc(need)
    assert st == OK
    return table + ids


# ---------------------------------------------------------------- spec pins
def test_figure_three_requests_share_the_system_prompt():
    """"LLM 推理优化：KV Cache、PagedAttention 与量化" §2.3 (3) figure: three
    requests with one system prompt point at blocks #7 #12 #3 and add private
    blocks #21 #8 / #5 #9 / #14 #2 — here found by content, not by an
    explicit fork."""
    _, kv = read_golden("prefix_sharing_figure.txt")
    d = dict(kv)
    bs = int(d["block_size"][0])
    prefix = [int(x) for x in d["prefix"]]
    suffixes = [[int(x) for x in v] for k, v in kv if k == "suffix"]
    pool = BlockPoolSpec(32, bs, _order(prefix + [i for s in suffixes for i in s], 32))
    cache = PrefixCacheSpec(pool)
    system = list(range(1000, 1000 + len(prefix) * bs))
    tables = []
    for r, suf in enumerate(suffixes):
        prompt = system + [2000 + 100 * r + i for i in range(len(suf) * bs)]
        table = _request(pool, cache, prompt)
        assert cache.register(prompt, table) == (OK, len(table))
        tables.append(table)
    for table, suf in zip(tables, suffixes):
        assert table == prefix + suf
    # three requests + the cache hold every prompt block
    assert all(pool.refcount[b] == len(suffixes) + 1 for b in prefix)
    assert all(pool.refcount[b] == 2 for s in suffixes for b in s)


def test_match_is_chained_through_the_parent():
    """A block's content alone does not match: block 1 of a prompt whose
    block 0 differs is a different prefix."""
    pool = BlockPoolSpec(16, 4)
    cache = PrefixCacheSpec(pool)
    a = [1, 2, 3, 4, 5, 6, 7, 8]
    ta = _request(pool, cache, a)
    cache.register(a, ta)
    b = [9, 9, 9, 9, 5, 6, 7, 8]           # same second block, other first block
    assert cache.match(b) == (OK, [])
    c = [9, 9, 9, 9, 0, 0, 0, 0]
    tc = _request(pool, cache, c)
    cache.register(c, tc)
    # block 0 of b is now cached (c's), block 1's content is cached under a's
    # chain only: the match must stop after block 0
    assert cache.match(b) == (OK, tc[:1])
    assert cache.match(a[:4] + [5, 6, 7, 0]) == (OK, ta[:1])
    assert cache.match(a + [1, 2]) == (OK, ta)   # the partial tail is never matched


def test_only_full_blocks_are_cached():
    pool = BlockPoolSpec(8, 4)
    cache = PrefixCacheSpec(pool)
    p = [1, 2, 3, 4, 5, 6]
    t = _request(pool, cache, p)
    assert cache.register(p, t) == (OK, 1)
    assert cache.num_cached() == 1
    assert pool.refcount[t[0]] == 2 and pool.refcount[t[1]] == 1


def test_eviction_takes_unreferenced_leaves_least_recent_first():
    pool = BlockPoolSpec(16, 2)
    cache = PrefixCacheSpec(pool)
    a, b = [1, 1, 2, 2, 3, 3], [1, 1, 7, 7]
    ta = _request(pool, cache, a)
    cache.register(a, ta)
    tb = _request(pool, cache, b)
    cache.register(b, tb)
    assert tb[0] == ta[0]
    pool.free(ta)
    pool.free(tb)
    # a's chain is older than b's block 1; block 0 is a parent until last
    st, out = cache.evict(10)
    assert st == OK and out == [ta[2], ta[1], tb[1], ta[0]]
    assert pool.num_free() == 16 and cache.num_cached() == 0
    # the freed blocks are reused first, last evicted on top
    assert pool.alloc(2) == (OK, [ta[0], tb[1]])


def test_referenced_blocks_are_never_evicted():
    pool = BlockPoolSpec(8, 2)
    cache = PrefixCacheSpec(pool)
    a = [1, 1, 2, 2]
    ta = _request(pool, cache, a)
    cache.register(a, ta)
    assert cache.evict(5) == (OK, [])        # the request still holds both
    pool.free(ta[1:])
    assert cache.evict(5) == (OK, [ta[1]])   # the parent is still in use
    assert cache.match(a) == (OK, ta[:1])


def test_register_stops_at_content_cached_elsewhere():
    pool = BlockPoolSpec(16, 2)
    cache = PrefixCacheSpec(pool)
    a = [1, 1, 2, 2]
    ta = _request(pool, cache, a)
    st, tb = pool.alloc(2)                   # computed again without a match
    assert cache.register(a, ta) == (OK, 2)
    assert cache.register(a, tb) == (OK, 0)
    assert cache.num_cached() == 2 and pool.refcount[tb[0]] == 1


class _UnchainedSpec(PrefixCacheSpec):
    """Mutant: keys ignore the parent."""

    def match(self, tokens):
        bs = self.pool.block_size
        table = []
        for i in range(len(tokens) // bs):
            hit = [b for (p, t), b in self.entries.items() if t == tuple(tokens[i * bs:(i + 1) * bs])]
            if not hit:
                break
            self.pool.refcount[hit[0]] += 1
            self._use(hit[0])
            table.append(hit[0])
        return OK, table


class _MruSpec(PrefixCacheSpec):
    """Mutant: evicts the most recently used first and ignores children."""

    def evict(self, n):
        out = []
        while len(out) < n:
            cand = [b for b in self.key_of if self.pool.refcount[b] == 1]
            if not cand:
                break
            b = max(cand, key=lambda x: self.last_use[x])
            key = self.key_of.pop(b)
            del self.entries[key]
            self.pool.free([b])
            out.append(b)
        return OK, out


@pytest.mark.parametrize("mutant", [_UnchainedSpec, _MruSpec])
def test_pins_catch_planted_mistakes(mutant, monkeypatch):
    import oracle.block_spec as bspec
    monkeypatch.setattr(bspec, "PrefixCacheSpec", mutant)
    monkeypatch.setitem(globals(), "PrefixCacheSpec", mutant)
    failed = 0
    for pin in (test_match_is_chained_through_the_parent,
                test_eviction_takes_unreferenced_leaves_least_recent_first):
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed >= 1


# ------------------------------------------------------- C++ against the spec
@pytest.mark.parametrize("seed,bs", [(1, 16), (2, 8), (3, 16)])
def test_cpp_prefix_cache_matches_spec(seed, bs):
    """Random requests drawn from a few shared system prompts: identical
    matches, registrations, evictions, tables, refcounts and free lists."""
    rng = np.random.Generator(np.random.PCG64(100 + seed))
    nb = 96
    order = rng.permutation(nb)
    spool = BlockPoolSpec(nb, bs, order)
    scache = PrefixCacheSpec(spool)
    impl = pkv.KVPool(nb, bs, order=order)
    systems = [list(rng.integers(0, 50, size=int(rng.integers(1, 5)) * bs)) for _ in range(4)]
    live = []   # (tokens, table)
    n_hits = 0
    for step in range(1500):
        op = int(rng.integers(0, 10))
        if op <= 4:
            sysp = systems[int(rng.integers(len(systems)))]
            cut = int(rng.integers(0, len(sysp) + 1))
            tokens = [int(x) for x in sysp[:cut]] + [int(x) for x in rng.integers(0, 3, size=int(rng.integers(0, 3 * bs)))]
            st, stab = scache.match(tokens)
            got = impl.prefix_match(tokens)
            assert got == stab
            n_hits += len(got)
            need = -(-len(tokens) // bs) - len(stab)
            st2, ids = spool.alloc(need)
            if st2 != OK:
                spool.free(stab)
                impl.free(got)
                with pytest.raises(pkv.KVError):
                    impl.alloc(need)
                continue
            assert impl.alloc(need) == ids
            live.append((tokens, stab + ids))
        elif op <= 6 and live:
            tokens, table = live[int(rng.integers(len(live)))]
            assert impl.prefix_register(tokens, table) == scache.register(tokens, table)[1]
        elif op <= 8 and live:
            tokens, table = live.pop(int(rng.integers(len(live))))
            assert spool.free(table) == OK
            impl.free(table)
        else:
            k = int(rng.integers(0, 6))
            assert impl.prefix_evict(k) == scache.evict(k)[1]
        assert impl.num_free() == spool.num_free()
        assert impl.num_cached() == scache.num_cached()
        if step % 50 == 0:
            assert [impl.refcount(b) for b in range(nb)] == spool.refcount
    assert n_hits > 50   # the workload really exercised matches
    for tokens, table in live:
        spool.free(table)
        impl.free(table)
    assert impl.prefix_evict(nb) == scache.evict(nb)[1]
    assert impl.num_free() == nb and impl.num_cached() == 0


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_cpp_eviction_tracks_forks_appends_and_beams(seed):
    """Cached blocks whose references also move through forks, appends
    (copy-on-write) and beam steps: the C++ cache evicts exactly the blocks
    the spec does, in the same order, with the same reference counts."""
    rng = np.random.Generator(np.random.PCG64(300 + seed))
    nb, bs = 128, 8
    order = rng.permutation(nb)
    spool = BlockPoolSpec(nb, bs, order)
    scache = PrefixCacheSpec(spool)
    impl = pkv.KVPool(nb, bs, order=order)
    systems = [list(rng.integers(0, 40, size=int(rng.integers(2, 6)) * bs)) for _ in range(3)]
    live = []   # [tokens, table]: the same ids on both sides
    extra = []  # references taken directly on cached blocks (no request)
    n_evicted = 0
    for step in range(1200):
        op = int(rng.integers(0, 13))
        if op <= 3 or not live:
            sysp = systems[int(rng.integers(len(systems)))]
            cut = int(rng.integers(0, len(sysp) + 1))
            tokens = [int(x) for x in sysp[:cut]] + [int(x) for x in rng.integers(0, 3, size=int(rng.integers(1, 2 * bs)))]
            st, stab = scache.match(tokens)
            assert impl.prefix_match(tokens) == stab
            need = -(-len(tokens) // bs) - len(stab)
            st2, ids = spool.alloc(need)
            if st2 != OK:
                spool.free(stab)
                impl.free(stab)
                continue
            assert impl.alloc(need) == ids
            live.append([tokens, stab + ids])
        elif op <= 5:
            tokens, table = live[int(rng.integers(len(live)))]
            assert impl.prefix_register(tokens, table) == scache.register(tokens, table)[1]
        elif op == 6:
            tokens, table = live[int(rng.integers(len(live)))]
            assert spool.fork(table) == OK
            impl.fork(table)
            live.append([list(tokens), list(table)])
        elif op == 7:
            tokens, table = live[int(rng.integers(len(live)))]
            before = list(table)
            st, slot, src, dst = spool.reserve_slot(table, len(tokens))
            if st != OK:
                continue
            t = np.full(len(before) + 1, -1, np.int32)
            t[:len(before)] = before
            assert impl.reserve_slot(t, len(before), len(tokens)) == (slot, len(table), src, dst)
            assert t[:len(table)].tolist() == table
            tokens.append(int(rng.integers(0, 3)))
        elif op == 8:
            k = int(rng.integers(1, min(3, len(live)) + 1))
            pick = sorted(rng.choice(len(live), size=k, replace=False).tolist())
            group = [live[i] for i in pick]
            parents = rng.integers(0, k, size=int(rng.integers(1, 4))).tolist()
            st, new = beam_reorder(spool, [g[1] for g in group], parents)
            assert st == OK
            cap = max(len(g[1]) for g in group)
            tabs = np.full((k, cap), -1, np.int32)
            for i, g in enumerate(group):
                tabs[i, :len(g[1])] = g[1]
            got, got_nb = impl.beam_reorder(tabs, np.array([len(g[1]) for g in group], np.int32), parents)
            assert [got[i, :got_nb[i]].tolist() for i in range(len(parents))] == new
            for i in reversed(pick):
                live.pop(i)
            live.extend([list(group[p][0]), list(t)] for p, t in zip(parents, new))
        elif op == 9:
            tokens, table = live.pop(int(rng.integers(len(live))))
            assert spool.free(table) == OK
            impl.free(table)
        elif op == 10:
            k = int(rng.integers(0, 8))
            got = impl.prefix_evict(k)
            assert got == scache.evict(k)[1]
            n_evicted += len(got)
        elif op == 11 and scache.key_of:
            # one more reference on cached blocks only the cache may hold
            ids = sorted(rng.choice(sorted(scache.key_of), size=min(3, len(scache.key_of)), replace=False).tolist())
            assert spool.fork(ids) == OK
            impl.fork(ids)
            extra.append(ids)
        elif op == 12 and extra:
            ids = extra.pop(int(rng.integers(len(extra))))
            assert spool.free(ids) == OK
            impl.free(ids)
        assert impl.num_free() == spool.num_free()
        assert impl.num_cached() == scache.num_cached()
        if step % 25 == 0:
            assert [impl.refcount(b) for b in range(nb)] == spool.refcount
    assert n_evicted >= 10   # eviction really ran against forked and beamed references
    for tokens, table in live:
        spool.free(table)
        impl.free(table)
    for ids in extra:
        spool.free(ids)
        impl.free(ids)
    assert impl.prefix_evict(nb) == scache.evict(nb)[1]
    assert impl.num_free() == nb and impl.num_cached() == 0


def test_cpp_register_rejects_dead_blocks():
    impl = pkv.KVPool(8, 8)
    ids = impl.alloc(1)
    impl.free(ids)
    with pytest.raises(pkv.KVError):
        impl.prefix_register(list(range(8)), ids)
    assert impl.num_cached() == 0
