"""Executable specification of the KV block pool's host bookkeeping — oracle.

Test infrastructure (see the package docstring): plain Python, written from
the pages' description, used to check the C++ block manager bit for bit.

What the pages fix ([T3] = "LLM 推理优化：KV Cache、PagedAttention 与量化"):
  * §2.2: the cache is cut into fixed-size blocks (16 tokens by default, 8 as a
    variant); a block table maps each sequence's logical blocks to physical
    ones.
  * §2.3 (1): blocks are taken from a fixed-capacity physical pool on demand
    (when a token is written), are returned to the pool as soon as the
    sequence ends and are reused first; the pool keeps an "unreferenced"
    counter per block; a full pool triggers preemption.
  * §2.3 (2): a beam fork copies only the block table; the physical blocks stay
    shared until a beam writes into one, at which point that block is copied
    and the writing beam's table is repointed (copy-on-write).
  * §2.3 (3): requests with a common prefix point their tables at the same
    physical blocks.

Policy choices where the pages are silent (each is a reading, fixed here so
that results are a single bit-exact answer):
  * free list is a LIFO stack; initially it pops in ascending id order, or in
    the order of a caller-given permutation; a freed block is pushed on top,
    so it is the first one reused ("立即回收…复用");
  * alloc(n) is all-or-nothing; on shortage nothing changes and OOM is
    reported (the pages' preemption trigger);
  * free(ids) decrements each reference; a block whose count reaches zero is
    pushed in the order given; a free that would take any count below zero
    changes nothing and reports DOUBLE_FREE;
  * fork(ids) adds one reference to each (live) block;
  * reserve_slot appends one token to a sequence: a full (or absent) last
    block -> a new block; a shared (refcount > 1) partial last block -> a new
    block, a (src, dst) copy pair, one reference dropped from src, the table
    repointed; otherwise the token goes into the last block.  Only a partial
    last block is ever copied.
"""
from __future__ import annotations

OK = 0
ERR_INVALID = 1
ERR_OOM = 2
ERR_DOUBLE_FREE = 3


class BlockPoolSpec:
    def __init__(self, num_blocks: int, block_size: int, order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("bad pool size")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.refcount = [0] * num_blocks
        order = list(range(num_blocks)) if order is None else [int(x) for x in order]
        if sorted(order) != list(range(num_blocks)):
            raise ValueError("order must be a permutation of 0..num_blocks-1")
        # top of stack = end of list; the first pop returns order[0]
        self.free_stack = list(reversed(order))

    # -- pool --------------------------------------------------------------
    def num_free(self) -> int:
        return len(self.free_stack)

    def alloc(self, n: int):
        if n < 0:
            return ERR_INVALID, []
        if n > len(self.free_stack):
            return ERR_OOM, []
        ids = [self.free_stack.pop() for _ in range(n)]
        for i in ids:
            self.refcount[i] = 1
        return OK, ids

    def free(self, ids):
        need = {}
        for i in ids:
            if not 0 <= i < self.num_blocks:
                return ERR_INVALID
            need[i] = need.get(i, 0) + 1
        for i, c in need.items():
            if self.refcount[i] < c:
                return ERR_DOUBLE_FREE
        for i in ids:
            self.refcount[i] -= 1
            if self.refcount[i] == 0:
                self.free_stack.append(i)
        return OK

    def fork(self, ids):
        for i in ids:
            if not 0 <= i < self.num_blocks or self.refcount[i] == 0:
                return ERR_INVALID
        for i in ids:
            self.refcount[i] += 1
        return OK

    # -- sequences ---------------------------------------------------------
    def reserve_slot(self, table: list, ctx_len: int):
        """Reserve the slot for token number ``ctx_len`` (0-based) of a
        sequence whose table is ``table`` (modified in place).

        Returns (status, slot, cow_src, cow_dst); cow_* are -1 without a copy.
        """
        bs = self.block_size
        if ctx_len < 0 or len(table) != -(-ctx_len // bs):
            return ERR_INVALID, -1, -1, -1
        off = ctx_len % bs
        if off == 0:
            st, ids = self.alloc(1)
            if st != OK:
                return st, -1, -1, -1
            table.append(ids[0])
            return OK, ids[0] * bs, -1, -1
        last = table[-1]
        if not 0 <= last < self.num_blocks or self.refcount[last] == 0:
            return ERR_INVALID, -1, -1, -1
        if self.refcount[last] > 1:
            st, ids = self.alloc(1)
            if st != OK:
                return st, -1, -1, -1
            new = ids[0]
            self.refcount[last] -= 1
            table[-1] = new
            return OK, new * bs + off, last, new
        return OK, last * bs + off, -1, -1


class PrefixCacheSpec:
    """Content-addressed cache of full blocks over a BlockPoolSpec.

    What the pages fix ([T3] §2.3 (3) and (1)): requests whose prompts share
    a prefix are detected by hashing block contents and point their tables at
    the same physical blocks; the pool keeps blocks that nothing references
    in LRU order.

    Readings (the pages give no more detail):
      * a block's identity is its parent block (the cached block holding the
        previous 16 tokens, -1 for the first) together with its own tokens:
        the key chains, so a match of block i implies a match of blocks
        0..i-1 (the K/V of a block depend on every earlier token).  Keys are
        compared exactly; the hash only places them (here: a dict);
      * only full blocks are cached and matched;
      * the cache holds one reference on every cached block, so a block
        outlives the requests that wrote it;
      * match(tokens) walks the prompt's full blocks from the start and stops
        at the first miss; every hit adds one reference (a fork) for the new
        request and counts as a use;
      * register(tokens, table) caches the table's full blocks in order; a
        block already cached under the same key is only marked used; the walk
        stops at a key cached under another block, or at a block cached under
        another key;
      * evict(n) releases up to n cached blocks that only the cache still
        references and that have no cached child (so a parent is never
        reused while a child's key names it), least recently used first;
        each is freed in the pool.
    """

    def __init__(self, pool: BlockPoolSpec):
        self.pool = pool
        self.entries = {}    # (parent, tokens) -> block
        self.key_of = {}     # block -> (parent, tokens)
        self.children = {}   # block -> cached children
        self.last_use = {}   # block -> use counter value
        self.clock = 0

    def _use(self, b):
        self.clock += 1
        self.last_use[b] = self.clock

    def num_cached(self) -> int:
        return len(self.key_of)

    def match(self, tokens):
        bs = self.pool.block_size
        table, parent = [], -1
        for i in range(len(tokens) // bs):
            b = self.entries.get((parent, tuple(tokens[i * bs:(i + 1) * bs])))
            if b is None:
                break
            self.pool.refcount[b] += 1
            self._use(b)
            table.append(b)
            parent = b
        return OK, table

    def register(self, tokens, table):
        bs = self.pool.block_size
        n = min(len(tokens) // bs, len(table))
        for b in table[:n]:
            if not 0 <= b < self.pool.num_blocks or self.pool.refcount[b] == 0:
                return ERR_INVALID, 0
        parent, done = -1, 0
        for i in range(n):
            b = table[i]
            key = (parent, tuple(tokens[i * bs:(i + 1) * bs]))
            have = self.entries.get(key)
            if have is None:
                if b in self.key_of:
                    break
                self.entries[key] = b
                self.key_of[b] = key
                self.children[b] = 0
                if parent >= 0:
                    self.children[parent] += 1
                self.pool.refcount[b] += 1
                self._use(b)
            elif have == b:
                self._use(b)
            else:
                break
            parent = b
            done += 1
        return OK, done

    def evict(self, n: int):
        if n < 0:
            return ERR_INVALID, []
        out = []
        while len(out) < n:
            cand = [b for b in self.key_of
                    if self.children[b] == 0 and self.pool.refcount[b] == 1]
            if not cand:
                break
            b = min(cand, key=lambda x: self.last_use[x])
            key = self.key_of.pop(b)
            del self.entries[key]
            del self.children[b]
            del self.last_use[b]
            if key[0] >= 0:
                self.children[key[0]] -= 1
            self.pool.free([b])
            out.append(b)
        return OK, out


def beam_reorder(pool: BlockPoolSpec, tables, parents):
    """One beam-search step over the pool's bookkeeping ([T3] §2.3 (2): a
    fork copies only the block table; the blocks stay shared until a beam
    writes into one).  New beam i continues old beam parents[i]: it gets a
    copy of that table and one more reference on each of its blocks; then
    every old beam's table is released, beam by beam in order (a block whose
    count reaches zero goes on the free list).  References are added before
    any is dropped, so a surviving block is never freed.  Returns
    (status, new_tables); nothing changes on an error."""
    n = len(tables)
    if any(not 0 <= p < n for p in parents):
        return ERR_INVALID, []
    for t in tables:
        for b in t:
            if not 0 <= b < pool.num_blocks or pool.refcount[b] == 0:
                return ERR_INVALID, []
    new = [list(tables[p]) for p in parents]
    for t in new:
        for b in t:
            pool.refcount[b] += 1
    for t in tables:
        for b in t:
            pool.refcount[b] -= 1
            if pool.refcount[b] == 0:
                pool.free_stack.append(b)
    return OK, new
