"""Pins for the oracle: what the pages and the mathematics fix, independent of it.

Each test below would fail under a plausible mistake in the oracle:
* slot translation (wrong divisor, table index, offset) -> worked example;
* attention (dropped scale, sign, transposed K/V, wrong head group, off-by-one
  length, wrong widening of bf16/f16) -> torch SDPA on the contiguous layout,
  closed forms, GQA via SDPA's own grouping, fp32/bf16/f16 agreement;
* allocator -> worked example, brute-force payload model and invariants,
  the free queue's order in closed form.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth
from oracle.allocator import INVALID, NO_FREE_BLOCK, OK, Allocator

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_block_table.txt")


def read_golden():
    spec = {"logical": []}
    for line in open(GOLDEN, encoding="utf-8"):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, *v = line.split()
        if k == "logical_block":
            spec["logical"].append(tuple(int(x) for x in v))
        else:
            spec[k] = int(v[0])
    return spec


# ---------------------------------------------------------------- worked example
def test_worked_example_slot_translation():
    g = read_golden()
    bs = g["block_size"]
    bt = [phys for (_, _, _, phys) in sorted(g["logical"])]
    for (j, first, last, phys) in g["logical"]:
        for t in range(first, last + 1):
            sl = oracle.slot(bt, bs, t)
            assert sl // bs == phys, (t, sl)
            assert sl % bs == t - first
    assert g["logical"][-1][2] == g["seq_len"] - 1


def test_worked_example_allocator_growth():
    g = read_golden()
    bs = g["block_size"]
    phys = [p for (_, _, _, p) in sorted(g["logical"])]
    nb = 16
    order = phys + [g["next_block"]] + [b for b in range(nb) if b not in phys + [g["next_block"]]]
    a = Allocator(nb, bs, order)
    assert a.seq_add(0) == OK
    st, slots, pairs = a.seq_append_slots(0, g["seq_len"])
    assert st == OK and pairs == []
    assert a.seq_block_table(0)[1] == phys
    free_before = a.stats()["free_blocks"]
    # Filling the rest of logical block 2 takes nothing from the free pool.
    for t in range(g["seq_len"], 3 * bs):
        st, sl, pr = a.seq_append_slots(0, 1)
        assert st == OK and pr == [] and sl == [phys[2] * bs + t % bs]
    assert a.stats()["free_blocks"] == free_before
    # The page's "36th token" is not where block 2 fills (stated reading).
    assert g["page_fill_token"] < 3 * bs
    # The next token takes the fresh block, appended to the table.
    st, sl, pr = a.seq_append_slots(0, 1)
    assert st == OK and pr == []
    assert a.seq_block_table(0)[1] == phys + [g["next_block"]]
    assert sl == [g["next_block"] * bs]
    assert a.stats()["free_blocks"] == free_before - 1


def test_worked_example_kv_append_lands_in_block_9():
    g = read_golden()
    b = synth.make_batch(synth.CONFIGS["tiny"])
    assert b.block_tables[0, :3].tolist() == [p for (_, _, _, p) in sorted(g["logical"])]
    k, v = b.k_pool.clone(), b.v_pool.clone()
    sm = np.full(4, -1, dtype=np.int64)
    # token index 35 of seq 0 goes to logical block 2 (physical 9), offset 3
    sm[0] = oracle.slot(b.block_tables[0], 16, 35)
    oracle.kv_append(k, v, b.k_new, b.v_new, sm)
    assert torch.equal(k[9, :, 3, :], b.k_new[0]) and torch.equal(v[9, :, 3, :], b.v_new[0])
    changed = (k != b.k_pool).any(dim=(1, 3)).nonzero().tolist()
    assert all(r == [9, 3] for r in changed)


def test_tiny_decode_step_allocates_only_where_the_last_block_is_full():
    """The tiny workload's decode step (lengths before the step 35, 16, 1, 50;
    the step appends token L of each sequence): only sequence 1, whose single
    block is full, takes a fresh block -- the front of the free pool -- while
    the others write into their partly filled last block at offset L mod 16
    (aiknowledge.cn 2.2.3: a new block only once the last one is full)."""
    b = synth.make_batch(synth.CONFIGS["tiny"])
    a = Allocator(b.num_blocks, 16, b.free_order)
    for s in range(4):
        assert a.seq_add(s) == OK and a.seq_append_slots(s, int(b.lens[s]))[0] == OK
    tables = [a.seq_block_table(s)[1] for s in range(4)]
    front, free_before = a.free[0], len(a.free)
    got = [a.seq_append_slots(s, 1) for s in range(4)]
    assert all(st == OK and pairs == [] for st, _, pairs in got)
    slots = [sl[0] for _, sl, _ in got]
    assert slots[0] == 9 * 16 + 3                                # block 9 of the worked example, offset 35 mod 16
    assert slots[1] == front * 16 and a.seq_block_table(1)[1] == tables[1] + [front]
    assert slots[2] == tables[2][0] * 16 + 1
    assert slots[3] == tables[3][3] * 16 + 50 % 16
    assert len(a.free) == free_before - 1
    assert [a.seq_block_table(s)[2] for s in range(4)] == [36, 17, 2, 51]


def test_block_copy_copies_only_that_block():
    b = synth.make_batch(synth.CONFIGS["tiny"])
    k, v = b.k_pool.clone(), b.v_pool.clone()
    oracle.block_copy(k, v, [(9, 30), (3, 31)])
    assert torch.equal(k[30], b.k_pool[9]) and torch.equal(v[31], b.v_pool[3])
    others = [i for i in range(32) if i not in (30, 31)]
    assert torch.equal(k[others], b.k_pool[others]) and torch.equal(v[others], b.v_pool[others])


# ------------------------------------------------------- contiguous == library SDPA
def scatter_contiguous(Kc, Vc, bs, NB, rng, pool_dtype):
    """Lay a contiguous [Hkv, L, D] K/V out block by block in a random pool."""
    Hkv, L, D = Kc.shape
    nb = -(-L // bs)
    blocks = rng.permutation(NB)[:nb]
    kp = torch.randn(NB, Hkv, bs, D).to(pool_dtype)
    vp = torch.randn(NB, Hkv, bs, D).to(pool_dtype)
    for j in range(nb):
        n = min(bs, L - j * bs)
        kp[blocks[j], :, :n, :] = Kc[:, j * bs:j * bs + n, :]
        vp[blocks[j], :, :n, :] = Vc[:, j * bs:j * bs + n, :]
    return kp, vp, blocks


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("Hq,Hkv,D,bs,L", [(4, 4, 64, 16, 35), (8, 2, 128, 32, 97),
                                            (16, 2, 64, 64, 200), (3, 1, 32, 16, 1)])
def test_contiguous_equals_sdpa(dtype, Hq, Hkv, D, bs, L):
    rng = np.random.default_rng(L * 7 + D)
    Kc = torch.randn(Hkv, L, D).to(dtype)
    Vc = torch.randn(Hkv, L, D).to(dtype)
    q = torch.randn(1, Hq, D).to(dtype)
    NB = -(-L // bs) + 5
    kp, vp, blocks = scatter_contiguous(Kc, Vc, bs, NB, rng, dtype)
    bt = np.full((1, len(blocks) + 2), -1, np.int32)
    bt[0, :len(blocks)] = blocks
    got = oracle.paged_attention(q, kp, vp, bt, [L])[0]
    ref = F.scaled_dot_product_attention(
        q.double()[:, :, None, :], Kc.double()[None], Vc.double()[None],
        enable_gqa=(Hq != Hkv))[0, :, 0, :]
    assert np.abs(got - ref.numpy()).max() < 1e-12


# ------------------------------------------------------------------ closed forms
def test_single_token_returns_its_value_exactly():
    D = 16
    k = torch.randn(3, 1, 4, D)
    v = torch.randn(3, 1, 4, D)
    q = torch.randn(1, 1, D)
    bt = np.array([[2, -1]], np.int32)
    out = oracle.paged_attention(q, k, v, bt, [1])[0, 0]
    assert np.array_equal(out, v[2, 0, 0].double().numpy())


def test_zero_query_gives_mean_of_values():
    D, L = 8, 11
    k = torch.randn(4, 1, 4, D)
    v = torch.randn(4, 1, 4, D)
    q = torch.zeros(1, 1, D)
    bt = np.array([[3, 0, 2]], np.int32)
    out = oracle.paged_attention(q, k, v, bt, [L])[0, 0]
    rows = [v[bt[0, t // 4], 0, t % 4].double() for t in range(L)]
    assert np.abs(out - torch.stack(rows).mean(0).numpy()).max() < 1e-15


def test_two_token_closed_form_pins_scale_and_sign():
    D = 64
    a, b0, b1 = 1.5, 2.0, -1.0
    q = torch.zeros(1, 1, D); q[0, 0, 5] = a
    k = torch.zeros(1, 1, 16, D); k[0, 0, 0, 5] = b0; k[0, 0, 1, 5] = b1
    v = torch.zeros(1, 1, 16, D); v[0, 0, 0, 0] = 1.0; v[0, 0, 1, 1] = 1.0
    out = oracle.paged_attention(q, k, v, np.array([[0]], np.int32), [2])[0, 0]
    x0, x1 = a * b0 / math.sqrt(D), a * b1 / math.sqrt(D)
    w1 = 1.0 / (1.0 + math.exp(x0 - x1))
    assert abs(out[0] - (1 - w1)) < 1e-15 and abs(out[1] - w1) < 1e-15
    # an explicit scale replaces 1/sqrt(D)
    out2 = oracle.paged_attention(q, k, v, np.array([[0]], np.int32), [2], scale=0.25)[0, 0]
    w1 = 1.0 / (1.0 + math.exp(0.25 * a * (b0 - b1)))
    assert abs(out2[1] - w1) < 1e-15


def test_dominant_key_selects_its_value():
    D, L = 32, 40
    k = torch.randn(3, 1, 16, D) * 0.01
    v = torch.randn(3, 1, 16, D)
    q = torch.zeros(1, 1, D); q[0, 0, 0] = 1.0
    k[1, 0, 7, 0] = 50.0 * math.sqrt(D)   # token 23 (block 1 of [2,1,0]) gets logit 50
    bt = np.array([[2, 1, 0]], np.int32)
    out = oracle.paged_attention(q, k, v, bt, [L])[0, 0]
    # every other weight is below e^-49 relative to the dominant one
    assert np.abs(out - v[1, 0, 7].double().numpy()).max() < 1e-15 + 40 * 5 * math.exp(-49)


def test_logit_shift_invariance():
    D, L = 16, 30
    k = torch.randn(2, 1, 16, D, dtype=torch.float32)
    v = torch.randn(2, 1, 16, D)
    q = torch.randn(1, 1, D)
    bt = np.array([[1, 0]], np.int32)
    base = oracle.paged_attention(q, k, v, bt, [L])[0, 0]
    # adding c * q / |q|^2 * sqrt(D) to every key adds c to every logit
    c = 7.0
    shift = (c * q[0, 0].double() / q[0, 0].double().pow(2).sum() * math.sqrt(D))
    k2 = (k.double() + shift).float()
    # float32 rounding of the shifted keys perturbs logits by ~1e-6; compare loosely
    out = oracle.paged_attention(q, k2, v, bt, [L])[0, 0]
    assert np.abs(out - base).max() < 1e-4


def test_zero_length_gives_zeros():
    k = torch.randn(2, 1, 16, 8); v = torch.randn(2, 1, 16, 8); q = torch.randn(2, 1, 8)
    out = oracle.paged_attention(q, k, v, np.array([[0], [1]], np.int32), [0, 5])
    assert np.all(out[0] == 0) and np.any(out[1] != 0)


# ------------------------------------------------------------- structural invariances
def test_prefix_stored_once_equals_copied():
    """A shared prefix read through shared blocks == the same prefix copied per sequence."""
    rng = np.random.default_rng(5)
    S, H, D, bs = 5, 2, 32, 16
    nbp = 3                                   # prefix = 3 full blocks = 48 tokens
    suf = rng.integers(1, 50, size=S)
    NB = 200
    k = torch.randn(NB, H, bs, D).to(torch.bfloat16)
    v = torch.randn(NB, H, bs, D).to(torch.bfloat16)
    q = torch.randn(S, H, D).to(torch.bfloat16)
    perm = rng.permutation(NB)
    shared = perm[:nbp]
    cur = nbp
    maxb = nbp + 5
    bt_shared = np.full((S, maxb), -1, np.int32)
    bt_copied = np.full((S, maxb), -1, np.int32)
    k2, v2 = k.clone(), v.clone()
    lens = nbp * bs + suf
    for s in range(S):
        nb = -(-int(lens[s]) // bs)
        own_prefix = perm[cur:cur + nbp]; cur += nbp
        k2[own_prefix] = k[shared]; v2[own_prefix] = v[shared]
        rest = perm[cur:cur + nb - nbp]; cur += nb - nbp
        bt_shared[s, :nb] = np.concatenate([shared, rest])
        bt_copied[s, :nb] = np.concatenate([own_prefix, rest])
    a = oracle.paged_attention(q, k, v, bt_shared, lens)
    b = oracle.paged_attention(q, k2, v2, bt_copied, lens)
    assert np.array_equal(a, b)


def test_physical_relabelling_is_invisible():
    b = synth.make_batch(synth.shrink(synth.CONFIGS["llama7b"], S=6, Hq=4, Hkv=4, len_uniform=(1, 90)))
    ref = oracle.paged_attention(b.q, b.k_pool, b.v_pool, b.block_tables, b.lens)
    rng = np.random.default_rng(11)
    perm = rng.permutation(b.num_blocks)          # new id of old block i is perm[i]
    inv = np.argsort(perm)
    k2 = b.k_pool[torch.from_numpy(inv)]
    v2 = b.v_pool[torch.from_numpy(inv)]
    bt2 = np.where(b.block_tables >= 0, perm[np.maximum(b.block_tables, 0)], -1).astype(np.int32)
    got = oracle.paged_attention(b.q, k2, v2, bt2, b.lens)
    assert np.array_equal(ref, got)


def test_gqa_equals_mha_with_repeated_kv_heads():
    b = synth.make_batch(synth.shrink(synth.CONFIGS["llama3_gqa_bs16"], S=3, Hq=8, Hkv=2,
                                      len_fixed=None, len_uniform=(1, 70)))
    gqa = oracle.paged_attention(b.q, b.k_pool, b.v_pool, b.block_tables, b.lens)
    G = 4
    kr = b.k_pool.repeat_interleave(G, dim=1)
    vr = b.v_pool.repeat_interleave(G, dim=1)
    mha = oracle.paged_attention(b.q, kr, vr, b.block_tables, b.lens)
    assert np.array_equal(gqa, mha)


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
def test_narrow_types_widen_exactly(dt):
    b = synth.make_batch(synth.shrink(synth.CONFIGS["tiny"], dtype={torch.bfloat16: "bf16", torch.float16: "f16"}[dt]))
    a = oracle.paged_attention(b.q, b.k_pool, b.v_pool, b.block_tables, b.lens)
    c = oracle.paged_attention(b.q.float(), b.k_pool.float(), b.v_pool.float(), b.block_tables, b.lens)
    assert np.array_equal(a, c)


def test_items_match_full_grid():
    b = synth.make_batch(synth.CONFIGS["tiny"])
    full = oracle.paged_attention(b.q, b.k_pool, b.v_pool, b.block_tables, b.lens, threads=3)
    items = [(3, 2), (0, 0), (1, 3)]
    part = oracle.paged_attention(b.q, b.k_pool, b.v_pool, b.block_tables, b.lens, items=items)
    for i, (s, h) in enumerate(items):
        assert np.array_equal(part[i], full[s, h])


def test_rejects_out_of_range_block():
    b = synth.make_batch(synth.CONFIGS["tiny"])
    bt = b.block_tables.copy(); bt[1, 0] = 99
    with pytest.raises(ValueError):
        oracle.paged_attention(b.q, b.k_pool, b.v_pool, bt, b.lens)


# ------------------------------------------------------ allocator: brute-force model
def check_state(a: Allocator, model: dict, data: dict):
    bs = a.block_size
    refs = [0] * a.num_blocks
    used = set()
    for sid, (bt, n) in a.seqs.items():
        assert sid in model
        assert len(bt) == -(-n // bs)                       # at most the last block partial
        assert len(set(bt)) == len(bt)
        for t in range(n):                                  # reads back its own tokens
            assert data.get(bt[t // bs] * bs + t % bs) == model[sid][t]
        assert len(model[sid]) == n
        for blk in bt:
            refs[blk] += 1
            used.add(blk)
    assert set(model) == set(a.seqs)
    assert refs == a.ref
    assert set(a.free).isdisjoint(used)
    assert len(a.free) + len(used) == a.num_blocks
    assert len(set(a.free)) == len(a.free)


def run_ops(a: Allocator, ops, bs):
    model, data = {}, {}
    payload = [0]
    for op in ops:
        snap = (list(a.free), list(a.ref), {k: (list(v[0]), v[1]) for k, v in a.seqs.items()})
        kind = op[0]
        if kind == "add":
            st = a.seq_add(op[1])
            if st == OK:
                model[op[1]] = []
        elif kind == "append":
            sid, n = op[1], op[2]
            pre = a.seqs.get(sid)
            pre_bt = list(pre[0]) if pre else None
            pre_len = pre[1] if pre else 0
            st, slots, pairs = a.seq_append_slots(sid, n)
            if st == OK:
                assert len(slots) == n and len(pairs) <= 1
                if pairs:
                    src, dst = pairs[0]
                    j = pre_len // bs
                    assert pre_bt[j] == src and pre_len % bs != 0        # only the written block
                    assert snap[1][src] > 1                               # and only if shared
                    for off in range(bs):
                        if src * bs + off in data:
                            data[dst * bs + off] = data[src * bs + off]
                for sl in slots:
                    payload[0] += 1
                    data[sl] = payload[0]
                    model[sid].append(payload[0])
        elif kind == "fork":
            st = a.seq_fork(op[1], op[2])
            if st == OK:
                model[op[2]] = list(model[op[1]])
        elif kind == "share":
            sid, donor, ntok = op[1], op[2], op[3]
            if donor in a.seqs and ntok <= a.seqs[donor][1]:
                blocks = a.seqs[donor][0][: -(-ntok // bs)]
            else:
                blocks = [0] * (-(-ntok // bs))
            st = a.seq_share_prefix(sid, blocks, ntok)
            if st == OK:   # the sharer sees whatever the shared blocks hold
                model[sid] = [data.get(blocks[t // bs] * bs + t % bs) for t in range(ntok)]
        else:
            st = a.seq_free(op[1])
            if st == OK:
                del model[op[1]]
        if st != OK:                                        # failed calls change nothing
            assert snap == (list(a.free), list(a.ref), {k: (list(v[0]), v[1]) for k, v in a.seqs.items()})
            assert st in (INVALID, NO_FREE_BLOCK)
        check_state(a, model, data)
    return model


def test_allocator_brute_force_model():
    n_fail = 0
    for seed in range(3000):
        nb = 4 + seed % 3
        a = Allocator(nb, 2, list(np.random.default_rng(seed).permutation(nb)))
        ops = synth.random_ops(seed, 8, max_seqs=4, max_append=4)
        run_ops(a, ops, 2)
        n_fail += a.alloc_failures
    assert n_fail > 0   # exhaustion paths were exercised


def test_allocator_exhaustion_is_atomic():
    a = Allocator(3, 4)
    assert a.seq_add(1) == OK
    assert a.seq_append_slots(1, 9)[0] == OK           # 3 blocks, 1 slot used of the last
    st, slots, pairs = a.seq_append_slots(1, 4)          # needs a 4th block
    assert st == NO_FREE_BLOCK and slots == [] and a.seqs[1][1] == 9
    assert a.stats() == dict(free_blocks=0, used_blocks=3, alloc_failures=1, cow_copies=0)


def test_free_queue_takes_from_the_front_and_frees_to_the_back_in_table_order():
    """The pages only say that a block is taken from the free pool when needed
    and returns to it when its sequence ends (aiknowledge.cn 2.2.2,
    openeuler.csdn.net explainer 8.2); the reading taken is a FIFO queue:
    take from the front, and a freed sequence's blocks join the back in
    block-table order, so a just-freed block is the last to be reused."""
    a = Allocator(6, 2, [5, 4, 3, 2, 1, 0])
    assert a.seq_add(0) == OK and a.seq_append_slots(0, 5)[0] == OK       # takes 5, 4, 3
    assert a.seq_block_table(0)[1] == [5, 4, 3]
    assert a.seq_add(1) == OK and a.seq_append_slots(1, 2)[0] == OK       # takes 2
    assert a.seq_free(0) == OK                                          # 5, 4, 3 join the back
    assert list(a.free) == [1, 0, 5, 4, 3]
    assert a.seq_add(2) == OK and a.seq_append_slots(2, 8)[0] == OK       # 1, 0 first, then 5, 4
    assert a.seq_block_table(2)[1] == [1, 0, 5, 4]
    st, slots, _ = a.seq_append_slots(2, 1)                              # token 8 opens a 5th block: 3
    assert st == OK and slots == [3 * 2 + 0]


def test_fork_then_append_copies_partial_block_once_per_writer():
    """Beam-style sharing: 4 beams of a sequence whose last block is partial."""
    bs = 64
    a = Allocator(40, bs)
    a.seq_add(0)
    a.seq_append_slots(0, 100)                            # 2 blocks, last holds 36
    for c in (1, 2, 3):
        assert a.seq_fork(0, c) == OK
    last = a.seqs[0][0][1]
    assert a.refcount(last) == 4
    copies = []
    for beam in (1, 2, 3, 0):
        st, slots, pairs = a.seq_append_slots(beam, 1)
        copies.append(pairs)
    # three writers copy; the last one owns the block alone and writes in place
    assert [len(p) for p in copies] == [1, 1, 1, 0]
    assert all(p[0][0] == last for p in copies[:3])
    assert a.refcount(last) == 1 and a.seqs[0][0][1] == last
    assert a.refcount(a.seqs[0][0][0]) == 4                # full blocks stay shared
    assert a.stats()["cow_copies"] == 3                     # the monitoring counter counts each copy


# ------------------------------------------------ chunks of new tokens (causal)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("Hq,Hkv,D,bs", [(4, 4, 64, 16), (8, 2, 128, 32)])
def test_chunk_equals_sdpa_with_causal_mask(dtype, Hq, Hkv, D, bs):
    """n new tokens at the end of a context of L: row i attends to tokens
    0 .. L-n+i -- torch SDPA on the contiguous layout with that mask."""
    rng = np.random.default_rng(D + bs)
    lens, ns = [40, 7, 100], [5, 7, 1]        # the second chunk is a whole prompt
    T = sum(ns)
    qs = np.concatenate([[0], np.cumsum(ns)]).astype(np.int32)
    q = torch.randn(T, Hq, D).to(dtype)
    NB = sum(-(-L // bs) for L in lens) + 4
    kp = torch.randn(NB, Hkv, bs, D).to(dtype)
    vp = torch.randn(NB, Hkv, bs, D).to(dtype)
    maxb = max(-(-L // bs) for L in lens)
    bt = np.full((3, maxb), -1, np.int32)
    perm = rng.permutation(NB)
    cur = 0
    ref = torch.zeros(T, Hq, D, dtype=torch.float64)
    for s, L in enumerate(lens):
        nb = -(-L // bs)
        bt[s, :nb] = perm[cur:cur + nb]
        cur += nb
        Kc = torch.cat([kp[bt[s, j]] for j in range(nb)], dim=1)[:, :L].double()   # [Hkv, L, D]
        Vc = torch.cat([vp[bt[s, j]] for j in range(nb)], dim=1)[:, :L].double()
        n = ns[s]
        mask = torch.arange(L)[None, :] <= (L - n + torch.arange(n))[:, None]       # [n, L]
        qq = q[qs[s]:qs[s + 1]].double().transpose(0, 1)[None]                     # [1, Hq, n, D]
        o = F.scaled_dot_product_attention(qq, Kc[None], Vc[None], attn_mask=mask, enable_gqa=(Hq != Hkv))
        ref[qs[s]:qs[s + 1]] = o[0].transpose(0, 1)
    got = oracle.paged_attention_chunk(q, kp, vp, bt, lens, qs)
    assert np.abs(got - ref.numpy()).max() < 1e-12


def test_chunk_of_one_token_is_decode():
    b = synth.make_batch(synth.shrink(synth.CONFIGS["llama3_gqa_bs16"], S=3, Hq=8, Hkv=2, D=64,
                                      len_fixed=None, len_uniform=(1, 90)))
    qs = np.arange(4, dtype=np.int32)
    a = oracle.paged_attention_chunk(b.q, b.k_pool, b.v_pool, b.block_tables, b.lens, qs)
    d = oracle.paged_attention(b.q, b.k_pool, b.v_pool, b.block_tables, b.lens)
    assert np.array_equal(a, d)


def test_chunk_last_row_sees_whole_context_first_row_sees_its_prefix():
    b = synth.make_batch(synth.shrink(synth.CONFIGS["llama7b"], S=1, Hq=2, Hkv=2, D=64, lens=[50], len_uniform=None))
    n = 6
    q = torch.randn(n, 2, 64)
    qs = np.array([0, n], np.int32)
    got = oracle.paged_attention_chunk(q, b.k_pool.float(), b.v_pool.float(), b.block_tables, b.lens, qs)
    for i in range(n):
        one = oracle.paged_attention(q[i:i + 1], b.k_pool.float(), b.v_pool.float(), b.block_tables[:1],
                                     [50 - n + i + 1])
        assert np.array_equal(got[i], one[0])


# ------------------------------------------------------------- FP8 E4M3 pools
def test_e4m3_table_matches_torch_float8():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    got = oracle.e4m3_table()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[~np.isnan(got)], ref[~np.isnan(ref)])


def e4m3_midpoints():
    """Every point halfway between two adjacent non-negative E4M3 values (from
    torch's decoding of the 256 codes), both signs: exact ties, which random
    inputs essentially never hit, so that ties-to-even is pinned too."""
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    v = np.unique(ref[np.isfinite(ref) & (ref >= 0)])
    mids = (v[:-1] + v[1:]) / 2
    return torch.from_numpy(np.concatenate([mids, -mids])).float()


@pytest.mark.parametrize("scale", [1.0, 0.125, 0.37])
def test_e4m3_quantize_matches_torch_cast_and_saturates(scale):
    g = torch.Generator().manual_seed(3)
    # times a power-of-two scale, each midpoint is still an exact tie after x * (1/scale)
    x = torch.cat([torch.randn(200000, generator=g) * 60, torch.tensor([0.0, -0.0, 1e-30, -1e-30, 447.9, 448.0,
                                                                         449.0, 463.9, 1e6, -1e6]),
                   e4m3_midpoints() * scale])
    codes = oracle.quantize_e4m3(x, scale)
    y = (x.float() * (torch.tensor(1.0, dtype=torch.float32) / torch.tensor(scale, dtype=torch.float32)))
    inside = y.abs() < 448
    ref = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes[inside.numpy()], ref[inside.numpy()])
    table = oracle.e4m3_table()
    out = ~inside.numpy()
    assert np.all(np.abs(table[codes[out]]) == 448.0)                    # saturated, sign kept
    assert np.array_equal(np.sign(table[codes[out]]), np.sign(y.numpy()[out]))


def test_fp8_append_places_torch_codes_at_the_slots():
    """Each new token's K and V, cast by torch's float8_e4m3fn after the
    x * fp32(1/scale) product, land at their slots (block slot // bs, offset
    slot % bs, every kv head); negative slots write nothing; every other code
    is untouched."""
    NB, Hkv, bs, D = 6, 2, 16, 32
    g = torch.Generator().manual_seed(11)
    kn = torch.randn(5, Hkv, D, generator=g) * 10
    vn = torch.randn(5, Hkv, D, generator=g) * 3
    slots = [3, -1, 40, 95, -7]
    ks, vs = 0.25, 0.0625
    kc = np.full((NB, Hkv, bs, D), 0x55, np.uint8)
    vc = np.full((NB, Hkv, bs, D), 0x55, np.uint8)
    oracle.kv_append_fp8(kc, vc, kn, vn, ks, vs, slots)
    ek = np.full_like(kc, 0x55)
    ev = np.full_like(vc, 0x55)
    for i, sl in enumerate(slots):
        if sl < 0:
            continue
        for codes, x, sc in ((ek, kn, ks), (ev, vn, vs)):
            y = x[i].float() * (torch.tensor(1.0) / torch.tensor(sc, dtype=torch.float32))
            codes[sl // bs, :, sl % bs, :] = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(kc, ek) and np.array_equal(vc, ev)


def test_fp8_attention_equals_attention_on_dequantized_values():
    """Pools of codes with power-of-two scales == the same values held as fp32."""
    b = synth.make_batch(synth.shrink(synth.CONFIGS["llama3_gqa_bs16"], S=3, Hq=8, Hkv=2, D=64,
                                      len_fixed=None, len_uniform=(1, 120)))
    ks, vs = 0.25, 2.0
    kc = oracle.quantize_e4m3(b.k_pool, ks)
    vc = oracle.quantize_e4m3(b.v_pool, vs)
    table = oracle.e4m3_table()
    kf = torch.from_numpy(table[kc] * ks).float()
    vf = torch.from_numpy(table[vc] * vs).float()
    a = oracle.paged_attention_kv(b.q, kc, vc, ks, vs, b.block_tables, b.lens)
    r = oracle.paged_attention(b.q.float(), kf, vf, b.block_tables, b.lens)
    assert np.array_equal(a, r)
