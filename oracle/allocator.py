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
