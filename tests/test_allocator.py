"""Product allocator (C++ in libpagedkv) vs the oracle allocator: bit-exact.

Both get the same seeded operation sequences; statuses, slots, copy-on-write
pairs, block tables, reference counts and counters must match after every op.
"""
import numpy as np
import pytest

import oracle
import synth
from paged_kv_cache_405_b200 import BlockAllocator
from oracle.allocator import INVALID, NO_FREE_BLOCK, OK, CachingAllocator


def compare(prod: BlockAllocator, orc: oracle.Allocator, sids):
    assert prod.stats() == orc.stats()
    for b in range(orc.num_blocks):
        assert prod.refcount(b) == orc.refcount(b)
    for sid in sids:
        assert prod.seq_block_table(sid) == orc.seq_block_table(sid)


def apply(a, op, bs):
    kind = op[0]
    if kind == "add":
        return a.seq_add(op[1])
    if kind == "append":
        return a.seq_append_slots(op[1], op[2])
    if kind == "fork":
        return a.seq_fork(op[1], op[2])
    if kind == "share":
        sid, donor, ntok = op[1], op[2], op[3]
        st, bt, n = a.seq_block_table(donor)
        blocks = bt[: -(-ntok // bs)] if st == OK and ntok <= n else [0] * (-(-ntok // bs))
        return a.seq_share_prefix(sid, blocks, ntok)
    return a.seq_free(op[1])


@pytest.mark.parametrize("seed0", [0, 1000, 2000])
def test_random_ops_bit_exact(seed0):
    for seed in range(seed0, seed0 + 700):
        nb = 4 + seed % 5
        bs = (1, 2, 4)[seed % 3]
        order = np.random.default_rng(seed).permutation(nb)
        prod = BlockAllocator(nb, bs, order)
        orc = oracle.Allocator(nb, bs, order)
        for op in synth.random_ops(seed, 10, max_seqs=4, max_append=6):
            r1 = apply(prod, op, bs)
            r2 = apply(orc, op, bs)
            assert r1 == r2, (seed, op, r1, r2)
            compare(prod, orc, range(4))


def test_worked_example_table():
    order = [7, 3, 9, 12] + [b for b in range(16) if b not in (7, 3, 9, 12)]
    a = BlockAllocator(16, 16, order)
    assert a.seq_add(0) == OK
    st, slots, pairs = a.seq_append_slots(0, 35)
    assert st == OK and pairs == [] and slots[0] == 112 and slots[34] == 146
    assert a.seq_block_table(0) == (OK, [7, 3, 9], 35)
    assert a.seq_append_slots(0, 13)[0] == OK
    assert a.seq_block_table(0)[1] == [7, 3, 9]
    st, slots, _ = a.seq_append_slots(0, 1)
    assert a.seq_block_table(0)[1] == [7, 3, 9, 12] and slots == [12 * 16]


def test_exhaustion_leaves_state_unchanged():
    a = BlockAllocator(3, 4)
    a.seq_add(1)
    assert a.seq_append_slots(1, 9)[0] == OK
    before = (a.stats(), a.seq_block_table(1))
    st, slots, pairs = a.seq_append_slots(1, 4)
    assert st == NO_FREE_BLOCK and slots == []
    after = (a.stats(), a.seq_block_table(1))
    assert after[1] == before[1]
    assert after[0]["alloc_failures"] == 1 and after[0]["free_blocks"] == 0


def test_invalid_calls():
    a = BlockAllocator(8, 4)
    assert a.seq_append_slots(5, 1)[0] == INVALID
    assert a.seq_free(5) == INVALID
    assert a.seq_add(1) == OK and a.seq_add(1) == INVALID
    assert a.seq_fork(1, 1) == INVALID and a.seq_fork(2, 3) == INVALID
    assert a.seq_share_prefix(1, [0], 2) == INVALID          # block 0 not in use
    assert a.refcount(-1) == -1 and a.refcount(8) == -1
    with pytest.raises(Exception):
        BlockAllocator(4, 4, [0, 1, 1, 2])


def test_shared_prefix_refcount():
    """A 512-token system prompt (32 blocks of 16) shared by 256 sequences."""
    b = synth.make_batch(synth.shrink(synth.CONFIGS["llama13b_prefix"], D=64, Hq=1, Hkv=1))
    a = BlockAllocator(b.num_blocks, 16, b.free_order)
    a.seq_add(-1)
    a.seq_append_slots(-1, 512)                              # the prompt, written once
    prefix = a.seq_block_table(-1)[1]
    assert prefix == b.prefix_blocks.tolist()
    for s in range(256):
        a.seq_add(s)
        assert a.seq_share_prefix(s, prefix, 512) == OK
    a.seq_free(-1)
    assert all(a.refcount(x) == 256 for x in prefix)
    for s in range(256):
        st, slots, pairs = a.seq_append_slots(s, int(b.lens[s]) - 512)
        assert st == OK and pairs == []                        # prefix ends on a block boundary
    for s in range(256):
        assert a.seq_block_table(s)[1] == b.block_tables[s][b.block_tables[s] >= 0].tolist()


def test_generator_handout_matches_allocator():
    b = synth.make_batch(synth.shrink(synth.CONFIGS["llama7b"], D=64, Hq=1, Hkv=1))
    a = BlockAllocator(b.num_blocks, b.shape.bs, b.free_order)
    for s in range(b.shape.S):
        a.seq_add(s)
        assert a.seq_append_slots(s, int(b.lens[s]))[0] == OK
        assert a.seq_block_table(s)[1] == b.block_tables[s][b.block_tables[s] >= 0].tolist()


def test_beam_fork_copy_on_write():
    """Four beams share a 100k-token parent (bs 64, last block holds 32 tokens)."""
    bs = 64
    nb = 1563 * 2 + 8
    a = BlockAllocator(nb, bs)
    o = oracle.Allocator(nb, bs)
    for x in (a, o):
        x.seq_add(0)
        assert x.seq_append_slots(0, 100_000)[0] == OK
        for c in (1, 2, 3):
            x.seq_fork(0, c)
    res = [[x.seq_append_slots(beam, 1) for beam in (1, 2, 3, 0)] for x in (a, o)]
    assert res[0] == res[1]
    assert [len(r[2]) for r in res[0]] == [1, 1, 1, 0]
    last = a.seq_block_table(0)[1][-1]
    assert all(r[2][0][0] == last for r in res[0][:3])
    assert a.stats() == o.stats() and a.stats()["cow_copies"] == 3


def test_batch_calls_equal_sequential_calls():
    """The batched step call equals one append call per sequence, in order,
    including several beams copying one shared partial block."""
    for seed in range(300):
        rng = np.random.default_rng(seed)
        nb, bs = 12 + seed % 7, (2, 4)[seed % 2]
        a1, a2 = BlockAllocator(nb, bs), BlockAllocator(nb, bs)
        o = oracle.Allocator(nb, bs)
        n0 = int(rng.integers(1, 7))
        for a in (a1, a2, o):
            a.seq_add(0)
            a.seq_append_slots(0, n0)
            for c in (1, 2, 3):
                a.seq_fork(0, c)
        ids = [int(x) for x in rng.integers(0, 4, size=int(rng.integers(1, 9)))]
        st, slots, pairs = a1.seq_append_slots_batch(ids)
        seq = [a2.seq_append_slots(i, 1) for i in ids]
        oseq = [o.seq_append_slots(i, 1) for i in ids]
        assert seq == oseq
        if all(r[0] == OK for r in seq):
            assert st == OK
            assert slots.tolist() == [r[1][0] for r in seq]
            assert [tuple(p) for p in pairs.tolist()] == [p for r in seq for p in r[2]]
        else:   # the batch fails as a whole with the first failing status, changing nothing
            assert st == next(r[0] for r in seq if r[0] != OK)
            assert slots.size == 0 and pairs.size == 0
        st, bt, lens = a1.seq_block_tables_batch([0, 1, 2, 3], 64)
        if all(r[0] == OK for r in seq):
            for i in range(4):
                t = a2.seq_block_table(i)
                assert bt[i][bt[i] >= 0].tolist() == t[1] and lens[i] == t[2]


def reference_groups(bt, lens, bs, min_size):
    """Plain restatement of the documented grouping rule."""
    n = len(lens)
    full = [min(max(int(L), 0) // bs, bt.shape[1]) for L in lens]
    runs, gap, i = [], None, 0
    while i < n:
        k, j = full[i], i + 1
        while j < n and k >= 1:
            c = 0
            while c < min(k, full[j]) and bt[j, c] == bt[i, c]:
                c += 1
            if c < 1:
                break
            k, j = c, j + 1
        if j - i >= min_size and k >= 1:
            if gap is not None:
                runs.append((gap, 0))
                gap = None
            runs.append((i, k * bs))
            i = j
        else:
            gap = i if gap is None else gap
            i += 1
    if gap is not None:
        runs.append((gap, 0))
    return [r[0] for r in runs] + ([n] if runs else []), [r[1] for r in runs]


def test_find_shared_prefix_groups_matches_rule():
    import paged_kv_cache_405_b200 as pkv
    for seed in range(400):
        rng = np.random.default_rng(seed)
        n, mb, bs = int(rng.integers(0, 14)), int(rng.integers(1, 7)), int(rng.choice([2, 4, 16]))
        bt = rng.integers(0, 4, size=(n, mb)).astype(np.int32)   # few ids: many coincidences
        lens = rng.integers(0, mb * bs + 1, size=n).astype(np.int32)
        ms = int(rng.integers(2, 5))
        gf, gs = pkv.find_shared_prefix_groups(bt, lens, bs, ms)
        rf, rs = reference_groups(bt, lens, bs, ms)
        assert gf.tolist() == rf and gs.tolist() == rs, seed


def test_shared_prefix_layout_is_one_group():
    import paged_kv_cache_405_b200 as pkv
    b = synth.make_batch(synth.shrink(synth.CONFIGS["llama13b_prefix"], D=64, Hq=1, Hkv=1))
    gf, gs = pkv.find_shared_prefix_groups(b.block_tables, b.lens, 16, 4)
    assert gf.tolist() == [0, 256] and gs.tolist() == [512]


def test_batch_calls_equal_sequential_calls_with_cached_blocks():
    """Caching mode: sequences given a prefix that ends part-way into a cached
    block copy it before writing (a cached block is never written in place);
    the batched step call equals one call per sequence, product and oracle,
    and on a pool too small for all the copies it fails as a whole, changing
    nothing but the failure count."""
    n_fail = 0
    for seed in range(400):
        rng = np.random.default_rng(seed)
        bs = (2, 4)[seed % 2]
        prompt = [int(x) for x in rng.integers(0, 3, size=3 * bs)]
        nb = 3 + int(rng.integers(0, 5))                   # the prompt's 3 blocks + a few free ones
        ntok = int(rng.integers(1, 3 * bs))                 # often ends inside a full, cached block
        a1 = BlockAllocator(nb, bs, prefix_caching=True)
        a2 = BlockAllocator(nb, bs, prefix_caching=True)
        o = CachingAllocator(nb, bs)
        for a in (a1, a2, o):
            assert a.seq_add_with_prompt(0, prompt)[0] == OK
            blocks = a.seq_block_table(0)[1][:-(-ntok // bs)]
            for s in (1, 2, 3):
                assert a.seq_add(s) == OK and a.seq_share_prefix(s, blocks, ntok) == OK
            if seed % 3:
                assert a.seq_free(0) == OK                  # the sharers (and the cache) hold the blocks
        before = ([a1.seq_block_table(s) for s in (1, 2, 3)], a1.stats(), a1.cache_stats())
        ids = [int(x) for x in rng.integers(1, 4, size=int(rng.integers(1, 7)))]
        st, slots, pairs = a1.seq_append_slots_batch(ids)
        seq, oseq = [], []
        for i in ids:                                       # one call per sequence, stopping at a failure
            seq.append(a2.seq_append_slots(i, 1))
            oseq.append(o.seq_append_slots(i, 1))
            if seq[-1][0] != OK:
                break
        assert seq == oseq, seed
        if all(r[0] == OK for r in seq):
            assert st == OK
            assert slots.tolist() == [r[1][0] for r in seq]
            assert [tuple(p) for p in pairs.tolist()] == [p for r in seq for p in r[2]]
            assert not ({r[1][0] // bs for r in seq} & set(o.key_of)), seed   # no write in a cached block
            for s in (1, 2, 3):
                assert a1.seq_block_table(s) == a2.seq_block_table(s)
            assert a1.cache_stats() == a2.cache_stats() == o.cache_stats()
        else:
            n_fail += 1
            assert st == NO_FREE_BLOCK and slots.size == 0 and pairs.size == 0
            stats = dict(before[1], alloc_failures=before[1]["alloc_failures"] + 1)
            assert ([a1.seq_block_table(s) for s in (1, 2, 3)], a1.stats(), a1.cache_stats()) == \
                (before[0], stats, before[2]), seed
    assert n_fail > 20     # the tight pools were exercised


def test_batched_appends_equal_single_calls_after_random_histories():
    """Random histories (append, fork, share, free), then one batched step
    over random live sequences: equal to one call per sequence (product and
    oracle) when those all succeed, else refused as a whole with nothing
    changed but the failure count."""
    n_ok = n_fail = 0
    for seed in range(600):
        rng = np.random.default_rng(seed)
        nb, bs = 4 + seed % 5, (1, 2, 4)[seed % 3]
        order = np.random.default_rng(seed).permutation(nb)
        p1, p2, o = BlockAllocator(nb, bs, order), BlockAllocator(nb, bs, order), oracle.Allocator(nb, bs, order)
        for op in synth.random_ops(seed, 10, max_seqs=4, max_append=6):
            r = [apply(a, op, bs) for a in (p1, p2, o)]
            assert r[0] == r[1] == r[2], (seed, op)
        live = [s for s in range(4) if s in o.seqs]
        if not live:
            continue
        ids = [live[int(i)] for i in rng.integers(0, len(live), size=int(rng.integers(1, 6)))]
        before = ([p1.seq_block_table(s) for s in range(4)], p1.stats())
        st, slots, pairs = p1.seq_append_slots_batch(ids)
        seq, oseq = [], []
        for i in ids:
            seq.append(p2.seq_append_slots(i, 1))
            oseq.append(o.seq_append_slots(i, 1))
            if seq[-1][0] != OK:
                break
        assert seq == oseq, seed
        if all(x[0] == OK for x in seq):
            n_ok += 1
            assert st == OK and slots.tolist() == [x[1][0] for x in seq], seed
            assert [tuple(p) for p in pairs.tolist()] == [p for x in seq for p in x[2]]
            assert [p1.seq_block_table(s) for s in range(4)] == [p2.seq_block_table(s) for s in range(4)]
        else:
            n_fail += 1
            assert st == NO_FREE_BLOCK and slots.size == 0, seed
            fails = dict(before[1], alloc_failures=before[1]["alloc_failures"] + 1)
            assert ([p1.seq_block_table(s) for s in range(4)], p1.stats()) == (before[0], fails), seed
    assert n_ok > 100 and n_fail > 10


def test_lengths_query_matches_the_tables_query():
    """seq_lens_batch gives each sequence's length (what the session's
    pre-step check reads) exactly as seq_block_tables_batch does, for
    sequences that share a prefix, were forked and grew; an unknown id is
    refused with nothing written."""
    a = BlockAllocator(64, 16)
    for sid, n in ((0, 35), (1, 0), (2, 16), (3, 100)):
        assert a.seq_add(sid) == OK
        if n:
            a.seq_append_slots(sid, n)
    assert a.seq_fork(0, 7) == OK
    a.seq_append_slots(7, 3)
    ids = [3, 0, 7, 1, 2, 0]
    st, lens = a.seq_lens_batch(ids)
    assert st == OK and lens.dtype == np.int64
    st2, _, lens2 = a.seq_block_tables_batch(ids, 16)
    assert st2 == OK and lens.tolist() == lens2.tolist() == [100, 35, 38, 0, 16, 35]
    st, lens = a.seq_lens_batch([0, 99])
    assert st == INVALID
    assert a.seq_lens_batch([])[0] == OK
