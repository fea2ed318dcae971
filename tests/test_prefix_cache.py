"""Automatic prefix caching: the oracle's caching allocator pinned by a
payload model in which every slot holds the whole prefix ending at its token
(a cached block may only serve an identical prefix), and the product's
allocator bit-exact against it."""
import numpy as np
import pytest

from oracle.allocator import OK, INVALID, NO_FREE_BLOCK, CachingAllocator


def caching_ops(seed, n_ops, max_seqs=5, vocab=3):
    """Prompts drawn from a few shared stems so that prefixes repeat."""
    rng = np.random.default_rng(seed)
    stems = [list(rng.integers(0, vocab, size=int(rng.integers(0, 9)))) for _ in range(3)]
    ops = []
    for _ in range(n_ops):
        k = rng.choice(["prompt", "prompt", "tokens", "tokens", "slots", "fork", "share", "free", "free"])
        a = int(rng.integers(0, max_seqs))
        if k == "prompt":
            toks = list(stems[int(rng.integers(0, 3))]) + list(rng.integers(0, vocab, size=int(rng.integers(0, 4))))
            ops.append(("prompt", a, [int(x) for x in toks]))
        elif k == "tokens":
            ops.append(("tokens", a, [int(x) for x in rng.integers(0, vocab, size=int(rng.integers(1, 5)))]))
        elif k == "slots":
            ops.append(("slots", a, int(rng.integers(1, 3))))
        elif k == "fork":
            ops.append(("fork", a, int(rng.integers(0, max_seqs))))
        elif k == "share":    # register a, then map it onto donor's first ntok tokens
            ops.append(("share", a, int(rng.integers(0, max_seqs)), int(rng.integers(1, 6))))
        else:
            ops.append(("free", a))
    return ops


def apply(a, op):
    k = op[0]
    if k == "prompt":
        return a.seq_add_with_prompt(op[1], op[2])
    if k == "tokens":
        return a.seq_append_tokens(op[1], op[2])
    if k == "slots":
        return a.seq_append_slots(op[1], op[2])
    if k == "fork":
        return a.seq_fork(op[1], op[2])
    if k == "share":
        sid, donor, ntok = op[1], op[2], op[3]
        st, bt, n = a.seq_block_table(donor)
        if st != OK or ntok > n:
            return INVALID
        st = a.seq_add(sid)
        if st != OK:
            return st
        st = a.seq_share_prefix(sid, bt[:-(-ntok // a.block_size)], ntok)
        if st != OK:
            a.seq_free(sid)
        return st
    return a.seq_free(op[1])


def check(a: CachingAllocator, model, data):
    """data[slot] is the whole prefix ending at the token held there: a
    token's K/V depends on every token before it, so a block may serve a
    sequence only if it was written under the same prefix."""
    bs = a.block_size
    refs = [0] * a.num_blocks
    for sid, (bt, n) in a.seqs.items():
        assert len(bt) == -(-n // bs) and len(model[sid]) == n
        for t in range(n):   # every sequence reads back its own tokens, each under its own prefix
            assert data.get(bt[t // bs] * bs + t % bs) == tuple(model[sid][:t + 1])
        for b in bt:
            refs[b] += 1
    assert refs == a.ref
    assert all(a.ref[b] == 0 and b in a.key_of for b in a.lru)
    used = {b for b in range(a.num_blocks) if a.ref[b] > 0}
    assert len(a.free) + len(a.lru) + len(used) == a.num_blocks
    assert not (set(a.free) & set(a.lru)) and not (set(a.free) & used)
    for key, b in a.cache.items():     # a cached block holds exactly its key's tokens
        assert a.key_of[b] == key
        assert [(data.get(b * bs + o) or (None,))[-1] for o in range(bs)] == list(key[1])


def run(a, ops):
    model, data = {}, {}
    for op in ops:
        r = apply(a, op)
        k = op[0]
        if k == "prompt" and r[0] == OK:
            sid, toks = op[1], op[2]
            n_cached, slots = r[1], r[2]
            assert n_cached % a.block_size == 0 and len(slots) == len(toks) - n_cached
            for i, sl in enumerate(slots):
                data[sl] = tuple(toks[:n_cached + i + 1])
            model[sid] = list(toks)
        elif k in ("tokens", "slots") and r[0] == OK:
            st, slots, pairs = r
            for src, dst in pairs:
                for o in range(a.block_size):
                    if src * a.block_size + o in data:
                        data[dst * a.block_size + o] = data[src * a.block_size + o]
            toks = op[2] if k == "tokens" else [None] * op[2]
            before = model[op[1]]
            for i, sl in enumerate(slots):
                data[sl] = tuple(before + list(toks[:i + 1]))
            model[op[1]] = before + list(toks)
        elif k == "fork" and r == OK:
            model[op[2]] = list(model[op[1]])
        elif k == "share" and r == OK:
            model[op[1]] = list(model[op[2]][:op[3]])
        elif k == "free" and r == OK:
            del model[op[1]]
        check(a, model, data)
    return model


def test_caching_oracle_payload_model():
    hits = 0
    for seed in range(1500):
        nb = 6 + seed % 5
        a = CachingAllocator(nb, 2)
        run(a, caching_ops(seed, 12))
        hits += a.hits
    assert hits > 100     # the shared stems were found again


def test_hit_counts_closed_form():
    bs, m = 4, 5
    prompt = list(range(m * bs + 2))          # 5 full blocks + 2 tokens
    a = CachingAllocator(64, bs)
    for k in range(4):
        st, n_cached, slots = a.seq_add_with_prompt(k, prompt)
        assert st == OK and n_cached == (0 if k == 0 else m * bs) and len(slots) == len(prompt) - n_cached
    assert a.cache_stats()["lookups"] == 4 * m and a.cache_stats()["hits"] == 3 * m
    assert all(a.refcount(b) == 4 for b in a.seq_block_table(0)[1][:m])


def test_freed_cached_blocks_are_evicted_oldest_first():
    bs = 2
    a = CachingAllocator(6, bs)
    a.seq_add_with_prompt(0, [1, 2, 3, 4])       # blocks x0, x1 cached
    a.seq_add_with_prompt(1, [5, 6, 7, 8])       # blocks y0, y1 cached
    x, y = a.seq_block_table(0)[1], a.seq_block_table(1)[1]
    a.seq_free(1)                                # y released first ...
    a.seq_free(0)                                # ... then x
    assert a.lru == y + x and a.stats()["free_blocks"] == 6
    st, n_cached, slots = a.seq_add_with_prompt(2, [9, 9, 9, 9, 9, 9])   # 2 free + 1 evicted
    assert st == OK and n_cached == 0 and a.cache_stats()["evictions"] == 1
    assert (CachingAllocator.ROOT, (5, 6)) not in a.cache          # y0 (released first) was evicted
    assert a.cache[(CachingAllocator.ROOT, (1, 2))] == x[0]         # x0 is still cached
    assert y[0] in a.seq_block_table(2)[1]                           # and its block was reused
    # the evicted block's key is gone: [5, 6, 7, 8] no longer hits
    st, n_cached, _ = a.seq_add_with_prompt(3, [5, 6, 7, 8])
    assert st == NO_FREE_BLOCK or n_cached == 0


def test_forked_sequence_keeps_registering_its_blocks():
    """A fork inherits the parent's token ids, so a block the child fills with
    known tokens is cached too: a later prompt equal to the child's tokens
    finds both full blocks."""
    a = CachingAllocator(16, 2)
    st, n_cached, _ = a.seq_add_with_prompt(0, [1, 2, 3])     # [1, 2] cached, [3] partly filled
    assert st == OK and n_cached == 0
    assert a.seq_fork(0, 1) == OK
    st, slots, pairs = a.seq_append_tokens(1, [4])             # the child's write copies the shared block
    assert st == OK and len(pairs) == 1
    st, n_cached, _ = a.seq_add_with_prompt(2, [1, 2, 3, 4, 5])
    assert st == OK and n_cached == 4


def test_prompt_that_does_not_fit_changes_nothing():
    a = CachingAllocator(3, 2)
    a.seq_add_with_prompt(0, [1, 2, 3, 4])
    before = (list(a.free), list(a.lru), dict(a.cache), a.cache_stats())
    st, n_cached, slots = a.seq_add_with_prompt(1, [1, 2, 5, 6, 7, 8, 9])
    assert st == NO_FREE_BLOCK and 1 not in a.seqs
    assert before == (list(a.free), list(a.lru), dict(a.cache), a.cache_stats())


def test_product_allocator_matches_caching_oracle():
    from paged_kv_cache_405_b200 import BlockAllocator
    for seed in range(1500):
        nb, bs = 6 + seed % 5, (2, 3)[seed % 2]
        order = np.random.default_rng(seed).permutation(nb)
        prod = BlockAllocator(nb, bs, order, prefix_caching=True)
        orc = CachingAllocator(nb, bs, order)
        for op in caching_ops(seed, 12):
            r1 = apply(prod, op)
            r2 = apply(orc, op)
            assert r1 == r2, (seed, op, r1, r2)
            assert prod.stats() == orc.stats()
            assert prod.cache_stats() == orc.cache_stats()
            for sid in range(5):
                assert prod.seq_block_table(sid) == orc.seq_block_table(sid)
            assert [prod.refcount(b) for b in range(nb)] == orc.ref


def test_caching_off_behaves_like_plain_allocator():
    from paged_kv_cache_405_b200 import BlockAllocator
    from oracle.allocator import Allocator
    a = BlockAllocator(8, 4)
    o = Allocator(8, 4)
    st, n_cached, slots = a.seq_add_with_prompt(0, list(range(10)))
    o.seq_add(0)
    assert (st, n_cached) == (OK, 0) and slots == o.seq_append_slots(0, 10)[1]
    a.seq_free(0)
    o.seq_free(0)
    assert a.stats() == o.stats() and a.cache_stats()["cached_blocks"] == 0
    st, n_cached, _ = a.seq_add_with_prompt(1, list(range(10)))
    assert n_cached == 0


def test_copy_of_a_cached_block_by_its_last_holder_frees_the_original():
    """A sequence holding a cached block with fewer of its tokens copies it
    before writing; when it was the block's last holder the original turns
    evictable at once, so the same call can take it back as a fresh block.
    The product allocator (single and batched calls) agrees with the oracle
    on every pool size, including the tightest."""
    from paged_kv_cache_405_b200 import BlockAllocator
    bs = 2
    for nb in range(3, 8):
        for n in range(1, 5):
            out = []
            for a in (BlockAllocator(nb, bs, prefix_caching=True), CachingAllocator(nb, bs)):
                assert a.seq_add_with_prompt(0, [1, 2, 3, 4])[0] == OK      # two cached blocks
                blocks = a.seq_block_table(0)[1]
                assert a.seq_add(1) == OK and a.seq_share_prefix(1, blocks, 3) == OK
                assert a.seq_free(0) == OK                                  # sequence 1 is the last holder
                st, slots, pairs = a.seq_append_slots(1, n)
                out.append((st, list(slots), [tuple(p) for p in pairs], a.seq_block_table(1), a.stats(),
                            a.cache_stats()))
            assert out[0] == out[1], (nb, n)
            assert out[1][0] == OK or nb == 3                              # only the 3-block pool runs short
            b = BlockAllocator(nb, bs, prefix_caching=True)                # batched: the same steps
            b.seq_add_with_prompt(0, [1, 2, 3, 4])
            b.seq_add(1)
            b.seq_share_prefix(1, b.seq_block_table(0)[1], 3)
            b.seq_free(0)
            st, slots, pairs = b.seq_append_slots_batch([1] * n)
            assert st == out[0][0]
            if st == OK:
                assert slots.tolist() == out[0][1] and [tuple(p) for p in pairs.tolist()] == out[0][2]


def test_batched_appends_equal_single_calls_after_random_histories():
    """Caching mode, random histories (prompts, token appends, forks, shared
    prefixes, frees), then one batched step over random live sequences: it
    equals one call per sequence in order (product and oracle) when those all
    succeed, and otherwise fails as a whole, changing nothing but the
    failure count."""
    from paged_kv_cache_405_b200 import BlockAllocator
    n_ok = n_fail = 0
    for seed in range(600):
        rng = np.random.default_rng(seed)
        nb, bs = 6 + seed % 5, (2, 3)[seed % 2]
        order = rng.permutation(nb)
        prod1 = BlockAllocator(nb, bs, order, prefix_caching=True)
        prod2 = BlockAllocator(nb, bs, order, prefix_caching=True)
        orc = CachingAllocator(nb, bs, order)
        for op in caching_ops(seed, 10):
            r = [apply(a, op) for a in (prod1, prod2, orc)]
            assert r[0] == r[1] == r[2], (seed, op)
        live = [s for s in range(5) if s in orc.seqs]
        if not live:
            continue
        ids = [live[int(i)] for i in rng.integers(0, len(live), size=int(rng.integers(1, 6)))]
        before = ([prod1.seq_block_table(s) for s in range(5)], prod1.stats(), prod1.cache_stats())
        st, slots, pairs = prod1.seq_append_slots_batch(ids)
        seq, oseq = [], []
        for i in ids:
            seq.append(prod2.seq_append_slots(i, 1))
            oseq.append(orc.seq_append_slots(i, 1))
            if seq[-1][0] != OK:
                break
        assert seq == oseq, seed
        if all(x[0] == OK for x in seq):
            n_ok += 1
            assert st == OK, seed
            assert slots.tolist() == [x[1][0] for x in seq]
            assert [tuple(p) for p in pairs.tolist()] == [p for x in seq for p in x[2]]
            assert [prod1.seq_block_table(s) for s in range(5)] == [prod2.seq_block_table(s) for s in range(5)]
            assert prod1.cache_stats() == prod2.cache_stats() == orc.cache_stats()
        else:
            n_fail += 1
            assert st == NO_FREE_BLOCK and slots.size == 0, seed
            after = ([prod1.seq_block_table(s) for s in range(5)], prod1.stats(), prod1.cache_stats())
            fails = dict(before[1], alloc_failures=before[1]["alloc_failures"] + 1)
            assert after == (before[0], fails, before[2]), seed
    assert n_ok > 100 and n_fail > 10
