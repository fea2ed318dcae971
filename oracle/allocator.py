"""Oracle block allocator -- TEST INFRASTRUCTURE ONLY (plain Python, slow).

Only the tests, the smoke check and the benchmark's CPU-baseline leg use this;
the product's allocator is separate C++ and shares nothing with it.

The steps follow the pages' statement of paged KV management:

* A fixed pool of equal-size blocks; a sequence takes a block from the free
  pool only when its last block is full, so at most its last block is partly
  filled (openeuler.csdn.net PagedAttention explainer, sections 4.1 and 4.3;
  agent.csdn.net PagedAttention blog, section 2.1).
* Each sequence keeps a block table, logical block -> physical block
  (explainer section 4.2; aiknowledge.cn "2.2 PagedAttention 与 KV Cache
  分页管理", sections 2.2.2-2.2.3).
* Blocks return to the free pool when a sequence finishes or is preempted
  (aiknowledge.cn 2.2.2).
* Several sequences may point at the same physical blocks (a shared prefix,
  explainer 6.1; aiknowledge.cn 2.2.3; or a forked sample/beam, agent.csdn.net
  blog 2.2); a per-block reference count says how many.
* Copy-on-write: a write into a block that others still reference first
  copies that one block to a fresh block; the writer continues on the copy,
  the original keeps serving the others (explainer 6.2).

Readings where the pages are silent: the free pool is a FIFO queue (allocate
from the front, free to the back, in block-table order); a call that cannot
complete changes nothing; only pool exhaustion counts as an allocation failure.
"""
from __future__ import annotations

import copy
from collections import deque

OK, INVALID, NO_FREE_BLOCK = 0, 1, 2


class Allocator:
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("bad pool")
        self.num_blocks = num_blocks
        self.block_size = block_size
        order = list(range(num_blocks)) if free_order is None else [int(b) for b in free_order]
        if sorted(order) != list(range(num_blocks)):
            raise ValueError("free_order must be a permutation of the pool")
        self.free = deque(order)
        self.ref = [0] * num_blocks
        self.seqs: dict[int, list] = {}  # seq id -> [block table (list), length]
        self.alloc_failures = 0
        self.cow_copies = 0

    # -- helpers -----------------------------------------------------------
    def _snapshot(self):
        return (copy.copy(self.free), list(self.ref), copy.deepcopy(self.seqs), self.cow_copies)

    def _restore(self, snap):
        self.free, self.ref, self.seqs, self.cow_copies = snap

    # -- operations --------------------------------------------------------
    def seq_add(self, sid: int) -> int:
        if sid in self.seqs:
            return INVALID
        self.seqs[sid] = [[], 0]
        return OK

    def seq_share_prefix(self, sid: int, blocks, ntok: int) -> int:
        """Map an empty sequence onto existing blocks holding ``ntok`` tokens."""
        blocks = [int(b) for b in blocks]
        if sid not in self.seqs or self.seqs[sid][1] != 0 or self.seqs[sid][0]:
            return INVALID
        if ntok < 0 or len(blocks) != -(-ntok // self.block_size):
            return INVALID
        if len(set(blocks)) != len(blocks):
            return INVALID
        for b in blocks:
            if b < 0 or b >= self.num_blocks or self.ref[b] == 0:
                return INVALID
        for b in blocks:
            self.ref[b] += 1
        self.seqs[sid] = [list(blocks), ntok]
        return OK

    def seq_fork(self, parent: int, child: int) -> int:
        if parent not in self.seqs or child in self.seqs:
            return INVALID
        bt, n = self.seqs[parent]
        for b in bt:
            self.ref[b] += 1
        self.seqs[child] = [list(bt), n]
        return OK

    def seq_append_slots(self, sid: int, n: int):
        """Reserve slots for ``n`` new tokens.  Returns (status, slots, cow_pairs)."""
        if sid not in self.seqs or n < 0:
            return INVALID, [], []
        snap = self._snapshot()
        bt, length = self.seqs[sid]
        bs = self.block_size
        slots, pairs = [], []
        for t in range(length, length + n):
            j = t // bs
            if j == len(bt):                      # last block full: take a fresh one
                if not self.free:
                    self._restore(snap)
                    self.alloc_failures += 1
                    return NO_FREE_BLOCK, [], []
                b = self.free.popleft()
                self.ref[b] = 1
                bt.append(b)
            elif self.ref[bt[j]] > 1:             # writing into a shared block: copy it first
                if not self.free:
                    self._restore(snap)
                    self.alloc_failures += 1
                    return NO_FREE_BLOCK, [], []
                b = self.free.popleft()
                pairs.append((bt[j], b))
                self.ref[bt[j]] -= 1
                self.ref[b] = 1
                bt[j] = b
                self.cow_copies += 1
            slots.append(bt[j] * bs + t % bs)
        self.seqs[sid][1] = length + n
        return OK, slots, pairs

    def seq_free(self, sid: int) -> int:
        if sid not in self.seqs:
            return INVALID
        bt, _ = self.seqs.pop(sid)
        for b in bt:
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free.append(b)
        return OK

    def seq_block_table(self, sid: int):
        if sid not in self.seqs:
            return INVALID, [], 0
        bt, n = self.seqs[sid]
        return OK, list(bt), n

    def stats(self):
        free = len(self.free)
        return dict(free_blocks=free, used_blocks=self.num_blocks - free,
                    alloc_failures=self.alloc_failures, cow_copies=self.cow_copies)

    def refcount(self, b: int) -> int:
        if b < 0 or b >= self.num_blocks:
            return -1
        return self.ref[b]


class CachingAllocator(Allocator):
    """The allocator with automatic prefix caching -- TEST INFRASTRUCTURE ONLY.

    Pages: with prefix caching the KV of a prompt prefix computed once is
    reused by later requests, which skip that part of the prefill
    (openeuler.csdn.net explainer 7.4); sequences can point at the same
    physical blocks (aiknowledge.cn 2.2.3); only byte-identical prefixes may
    share (aiknowledge.cn 2.2.8); the hit rate is worth monitoring (2.2.13).

    Readings where the pages are silent:
    * only full blocks are cached; a block's key is (key node of the block
      before it, its bs token ids), so two blocks share a key exactly when
      their whole prefixes are identical; the first block's parent is the root;
    * every registration gets a fresh node id; a lookup walks a prompt's full
      blocks from the root and stops at the first miss;
    * a block becomes cached when it fills while its sequence's token ids are
      known and its parent block is cached on the sequence's chain; if the key
      is already cached (computed elsewhere) the new block is not registered
      and the chain of that sequence stops;
    * when a cached block's count drops to zero it is kept (evictable, at the
      back of an LRU list) instead of returning to the free queue; a fresh
      block comes from the free queue first, then by evicting the front of
      the LRU list, which drops its key;
    * a cached block is never written in place: a sequence that holds one
      with fewer of its tokens (a prefix shared part-way into it) copies it
      before writing, as a writer of a shared block does;
    * lookups/hits are counted in full blocks of the prompts looked up.
    """

    ROOT = -1

    def __init__(self, num_blocks, block_size, free_order=None):
        super().__init__(num_blocks, block_size, free_order)
        self.key_of = {}           # block -> key (cached blocks)
        self.node_of = {}          # block -> node id (cached blocks)
        self.cache = {}            # key -> block
        self.lru = []              # evictable cached blocks, oldest first
        self.next_node = 0
        self.tokens = {}           # sid -> list of token ids (None if unknown)
        self.chain = {}            # sid -> node id of its last cached block (ROOT, or None if broken)
        self.lookups = 0
        self.hits = 0
        self.evictions = 0

    def _snapshot(self):
        return (super()._snapshot(), dict(self.key_of), dict(self.node_of), dict(self.cache), list(self.lru),
                self.next_node, copy.deepcopy(self.tokens), dict(self.chain), self.evictions)

    def _restore(self, snap):
        (base, self.key_of, self.node_of, self.cache, self.lru, self.next_node, self.tokens, self.chain,
         self.evictions) = snap
        super()._restore(base)

    def _take(self):
        if self.free:
            return self.free.popleft()
        if self.lru:
            b = self.lru.pop(0)
            del self.cache[self.key_of.pop(b)]
            del self.node_of[b]
            self.evictions += 1
            return b
        return None

    def _release(self, b):
        self.ref[b] -= 1
        if self.ref[b] == 0:
            if b in self.key_of:
                self.lru.append(b)
            else:
                self.free.append(b)

    def stats(self):
        free = len(self.free) + len(self.lru)
        return dict(free_blocks=free, used_blocks=self.num_blocks - free, alloc_failures=self.alloc_failures,
                    cow_copies=self.cow_copies)

    def cache_stats(self):
        return dict(lookups=self.lookups, hits=self.hits, cached_blocks=len(self.cache),
                    evictable_blocks=len(self.lru), evictions=self.evictions)

    # -- operations --------------------------------------------------------
    def seq_add(self, sid):
        st = super().seq_add(sid)
        if st == OK:
            self.tokens[sid] = []
            self.chain[sid] = self.ROOT
        return st

    def seq_share_prefix(self, sid, blocks, ntok):
        st = super().seq_share_prefix(sid, blocks, ntok)
        if st == OK:
            self.tokens[sid] = None       # token ids unknown: never registers blocks
            self.chain[sid] = None
        return st

    def seq_fork(self, parent, child):
        st = super().seq_fork(parent, child)
        if st == OK:
            t = self.tokens[parent]
            self.tokens[child] = None if t is None else list(t)
            self.chain[child] = self.chain[parent]
        return st

    def seq_free(self, sid):
        if sid not in self.seqs:
            return INVALID
        bt, _ = self.seqs.pop(sid)
        for b in bt:
            self._release(b)
        self.tokens.pop(sid, None)
        self.chain.pop(sid, None)
        return OK

    def seq_append_slots(self, sid, n):
        """Appending without token ids: the sequence's tokens become unknown."""
        st, slots, pairs = self._append(sid, [None] * n if n >= 0 else None)
        return st, slots, pairs

    def seq_append_tokens(self, sid, toks):
        return self._append(sid, list(toks))

    def _append(self, sid, toks):
        if sid not in self.seqs or toks is None:
            return INVALID, [], []
        snap = self._snapshot()
        bt, length = self.seqs[sid]
        bs = self.block_size
        slots, pairs = [], []
        for k, tok in enumerate(toks):
            t = length + k
            j = t // bs
            if j == len(bt):
                b = self._take()
                if b is None:
                    self._restore(snap)
                    self.alloc_failures += 1
                    return NO_FREE_BLOCK, [], []
                self.ref[b] = 1
                bt.append(b)
            elif self.ref[bt[j]] > 1 or bt[j] in self.key_of:   # shared, or cached: copy first
                b = self._take()
                if b is None:
                    self._restore(snap)
                    self.alloc_failures += 1
                    return NO_FREE_BLOCK, [], []
                pairs.append((bt[j], b))
                self._release(bt[j])
                self.ref[b] = 1
                bt[j] = b
                self.cow_copies += 1
            slots.append(bt[j] * bs + t % bs)
            tl = self.tokens[sid]
            if tl is not None:
                if tok is None:
                    self.tokens[sid] = None
                    self.chain[sid] = None
                else:
                    tl.append(tok)
                    if t % bs == bs - 1:          # block j just filled
                        self._register(sid, bt[j], tl[j * bs:(j + 1) * bs])
        self.seqs[sid][1] = length + len(toks)
        return OK, slots, pairs

    def _register(self, sid, b, block_toks):
        parent = self.chain[sid]
        if parent is None:
            return
        key = (parent, tuple(block_toks))
        if key in self.cache:               # computed elsewhere already: this chain stops
            self.chain[sid] = None
            return
        node = self.next_node
        self.next_node += 1
        self.cache[key] = b
        self.key_of[b] = key
        self.node_of[b] = node
        self.chain[sid] = node

    def seq_add_with_prompt(self, sid, toks):
        """Register a sequence with prompt ``toks``: reuse the longest run of
        cached full blocks, reserve slots for the remaining tokens.  Returns
        (status, number of cached tokens, slots of the remaining tokens)."""
        if sid in self.seqs:
            return INVALID, 0, []
        toks = list(toks)
        bs = self.block_size
        snap = self._snapshot()
        node, hit_blocks = self.ROOT, []
        for j in range(len(toks) // bs):
            b = self.cache.get((node, tuple(toks[j * bs:(j + 1) * bs])))
            if b is None:
                break
            hit_blocks.append(b)
            node = self.node_of[b]
        for b in hit_blocks:
            if self.ref[b] == 0:
                self.lru.remove(b)
            self.ref[b] += 1
        n_cached = len(hit_blocks) * bs
        self.seqs[sid] = [list(hit_blocks), n_cached]
        self.tokens[sid] = toks[:n_cached]
        self.chain[sid] = node
        st, slots, _ = self._append(sid, toks[n_cached:])   # counts its own allocation failure
        if st != OK:
            self._restore(snap)
            return st, 0, []
        self.lookups += len(toks) // bs
        self.hits += len(hit_blocks)
        return OK, n_cached, slots
