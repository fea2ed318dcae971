"""DecodeSession's host side on CPU tensors: a failed ``add`` leaves no
sequence behind (the id can be registered again) and gives back every block
it took or mapped."""
import pytest
import torch

import paged_kv_cache_405_b200 as pkv


def session(num_blocks=4, bs=16):
    k = torch.zeros(num_blocks, 1, bs, 64, dtype=torch.bfloat16)
    return pkv.DecodeSession(k, k.clone(), 1, 8, max_batch=2)


def test_add_that_runs_out_of_blocks_registers_nothing():
    ss = session()
    with pytest.raises(pkv.PagedKVError):
        ss.add(0, 5 * 16)                          # needs 5 of 4 blocks
    assert ss.alloc.stats()["free_blocks"] == 4
    assert ss.add(0, 16) == list(range(0, 16))    # the id is free again; block 0 first
    assert ss.table(0) == ([0], 16)


def test_add_with_a_bad_prefix_registers_nothing_and_keeps_refcounts():
    ss = session()
    ss.add(0, 20)                                  # blocks 0, 1
    prompt, _ = ss.table(0)
    with pytest.raises(pkv.PagedKVError):
        ss.add(1, 3, shared_prefix=prompt, prefix_tokens=40)   # 40 tokens need 3 blocks, not 2
    assert [ss.alloc.refcount(b) for b in prompt] == [1, 1]
    with pytest.raises(pkv.PagedKVError):
        ss.add(1, 3 * 16, shared_prefix=prompt, prefix_tokens=32)   # mapped, then out of blocks
    assert [ss.alloc.refcount(b) for b in prompt] == [1, 1]
    assert ss.alloc.stats()["free_blocks"] == 2
    assert ss.add(1, 0, shared_prefix=prompt, prefix_tokens=32) == []
    assert [ss.alloc.refcount(b) for b in prompt] == [2, 2]


def test_plan_fails_before_reserving_anything():
    """A step that names an unknown sequence, or would grow a sequence past
    max_blocks_per_seq, raises with every table and the free pool unchanged."""
    k = torch.zeros(8, 1, 16, 64, dtype=torch.bfloat16)
    ss = pkv.DecodeSession(k, k.clone(), 1, 2, max_batch=4)          # at most 2 blocks per sequence
    ss.add(0, 10)
    ss.add(1, 32)                                                    # full: 2 blocks
    before = (ss.table(0), ss.table(1), ss.alloc.stats())
    with pytest.raises(pkv.PagedKVError):
        ss.plan([0, 7])                                              # unknown sequence 7
    with pytest.raises(pkv.PagedKVError):
        ss.plan([0, 1])                                              # token 32 of seq 1 needs a 3rd block
    with pytest.raises(pkv.PagedKVError):
        ss.plan_chunk([0], [23])                                     # 10 + 23 tokens need 3 blocks
    assert (ss.table(0), ss.table(1), ss.alloc.stats()) == before
    p = ss.plan([0], write=[0, 0])                                   # two tokens of seq 0 still fit
    assert p.lens.tolist() == [12] and ss.table(0)[1] == 12
    p = ss.plan_chunk([0], [20])                                     # exactly 32 tokens: fits
    assert p.lens.tolist() == [32]


def test_session_plans_match_the_oracle_allocator_on_random_steps():
    """Random mixes of add / fork / free / plan / plan_chunk: every plan's
    slots, copy pairs, padded tables and lengths equal what the oracle
    allocator gives for the same calls one token at a time; a step that
    would outgrow max_blocks_per_seq is refused and changes nothing."""
    import numpy as np

    import oracle
    bs, max_blocks, NB = 16, 4, 400
    for seed in range(60):
        rng = np.random.default_rng(seed)
        order = rng.permutation(NB).tolist()
        k = torch.zeros(NB, 1, bs, 64, dtype=torch.bfloat16)
        ss = pkv.DecodeSession(k, k.clone(), 1, max_blocks, free_order=order, max_batch=16, share_prefixes=False)
        orc = oracle.Allocator(NB, bs, order)
        live, next_id = [], 0
        for _ in range(40):
            op = rng.choice(["add", "add", "fork", "free", "plan", "plan", "chunk"])
            if op == "add" or not live:
                n = int(rng.integers(0, max_blocks * bs + 1))
                assert ss.add(next_id, n) == (orc.seq_add(next_id), orc.seq_append_slots(next_id, n))[1][1]
                live.append(next_id)
                next_id += 1
            elif op == "fork":
                p = live[int(rng.integers(len(live)))]
                ss.fork(p, next_id)
                orc.seq_fork(p, next_id)
                live.append(next_id)
                next_id += 1
            elif op == "free":
                sid = live.pop(int(rng.integers(len(live))))
                ss.free(sid)
                orc.seq_free(sid)
            else:
                ids = [live[i] for i in sorted(rng.choice(len(live), size=int(rng.integers(1, len(live) + 1)),
                                                          replace=False))]
                n_new = [1] * len(ids) if op == "plan" else rng.integers(1, 4, size=len(ids)).tolist()
                lens = {s: orc.seq_block_table(s)[2] for s in ids}
                too_long = any(-(-(lens[s] + n) // bs) > max_blocks for s, n in zip(ids, n_new))
                before = [ss.table(s) for s in ids]
                if too_long:
                    with pytest.raises(pkv.PagedKVError):
                        ss.plan(ids) if op == "plan" else ss.plan_chunk(ids, n_new)
                    assert [ss.table(s) for s in ids] == before
                    continue
                p = ss.plan(ids) if op == "plan" else ss.plan_chunk(ids, n_new)
                slots, pairs = [], []
                for s, n in zip(ids, n_new):
                    st, sl, pr = orc.seq_append_slots(s, n)
                    assert st == 0
                    slots += sl
                    pairs += pr
                assert p.slot_mapping.tolist() == slots, seed
                assert [tuple(x) for x in p.cow_pairs.tolist()] == [tuple(x) for x in pairs], seed
                for i, s in enumerate(ids):
                    _, t, L = orc.seq_block_table(s)
                    assert p.lens[i] == L and p.block_tables[i].tolist() == t + [-1] * (max_blocks - len(t))


def test_caching_session_matches_the_oracle_on_random_steps():
    """A DecodeSession with prefix caching: random prompts (a few shared
    stems), decode steps, forks and frees give the caching oracle's cached
    token counts, slots, copy pairs, tables and cache counters."""
    import numpy as np

    from oracle.allocator import CachingAllocator
    bs, max_blocks, NB = 16, 8, 48
    for seed in range(40):
        rng = np.random.default_rng(seed)
        stems = [rng.integers(0, 4, size=int(rng.integers(0, 3 * bs))).tolist() for _ in range(3)]
        order = rng.permutation(NB).tolist()
        k = torch.zeros(NB, 1, bs, 64, dtype=torch.bfloat16)
        ss = pkv.DecodeSession(k, k.clone(), 1, max_blocks, free_order=order, max_batch=8, share_prefixes=False,
                               prefix_caching=True)
        orc = CachingAllocator(NB, bs, order)
        live, next_id = [], 0
        for _ in range(30):
            op = rng.choice(["prompt", "prompt", "plan", "plan", "fork", "free"])
            if op == "prompt" or not live:
                toks = stems[int(rng.integers(3))] + rng.integers(0, 4, size=int(rng.integers(1, bs))).tolist()
                st, n_cached, oslots = orc.seq_add_with_prompt(next_id, toks)
                if st != 0:
                    with pytest.raises(pkv.PagedKVError):
                        ss.add_prompt(next_id, toks)
                    continue
                got_n, got_slots = ss.add_prompt(next_id, toks)
                assert (got_n, got_slots.tolist()) == (n_cached, oslots), seed
                live.append(next_id)
                next_id += 1
            elif op == "fork":
                p = live[int(rng.integers(len(live)))]
                ss.fork(p, next_id)
                orc.seq_fork(p, next_id)
                live.append(next_id)
                next_id += 1
            elif op == "free":
                sid = live.pop(int(rng.integers(len(live))))
                ss.free(sid)
                orc.seq_free(sid)
            else:
                ids = [live[i] for i in sorted(rng.choice(len(live), size=int(rng.integers(1, len(live) + 1)),
                                                          replace=False))]
                lens = {s: orc.seq_block_table(s)[2] for s in ids}
                need = sum(1 for s in ids if lens[s] % bs == 0) + len(ids)
                if any(-(-(lens[s] + 1) // bs) > max_blocks for s in ids) or need > orc.stats()["free_blocks"]:
                    continue                                  # keep to steps both sides can take
                p = ss.plan(ids)
                slots, pairs = [], []
                for s in ids:
                    st, sl, pr = orc.seq_append_slots(s, 1)
                    assert st == 0
                    slots += sl
                    pairs += pr
                assert p.slot_mapping.tolist() == slots and [tuple(x) for x in p.cow_pairs.tolist()] == pairs, seed
                for i, s in enumerate(ids):
                    _, t, L = orc.seq_block_table(s)
                    assert p.lens[i] == L and p.block_tables[i].tolist() == t + [-1] * (max_blocks - len(t))
            assert ss.cache_stats() == orc.cache_stats(), seed


def test_output_copy_overlap_needs_input_copy_overlap():
    """The output copies may leave the caller's stream only when the input
    copies do (the step's C call keys the output stream's wait on the input
    side's event); both modes construct, one without the other is refused."""
    k = torch.zeros(4, 1, 16, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="needs overlap_input_copies"):
        pkv.DecodeSession(k, k.clone(), 1, 8, max_batch=2, overlap_input_copies=False, overlap_output_copies=True)
    for ins, outs in ((True, True), (True, False), (False, False)):
        ss = pkv.DecodeSession(k, k.clone(), 1, 8, max_batch=2, overlap_input_copies=ins,
                               overlap_output_copies=outs)
        assert (ss.overlap_input_copies, ss.overlap_output_copies) == (ins, outs)
