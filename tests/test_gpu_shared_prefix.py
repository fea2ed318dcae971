"""GPU parity of the shared-prefix decode (pkv_paged_attention_decode_shared)
against the oracle, and against the plain decode on the same inputs.

A system prompt stored once and referenced by many sequences
(openeuler.csdn.net PagedAttention explainer 6.1; aiknowledge.cn "2.2
PagedAttention 与 KV Cache 分页管理" 2.2.3) must give the same attention as if
every sequence had its own copy; the prefix pass only changes how often the
shared blocks are read."""
import numpy as np
import pytest
import torch

import synth
from gpu_helpers import TOL, max_err, oracle_attention, to_dev

pytestmark = pytest.mark.gpu


def pkv():
    import paged_kv_cache_405_b200 as m
    return m


def run_shared(batch, gf, gs, P=0, max_group=None, max_shared=None):
    d = to_dev(batch)
    out = torch.full_like(d["q"], float("nan"))
    gft = torch.as_tensor(np.asarray(gf, np.int32)).cuda()
    gst = torch.as_tensor(np.asarray(gs, np.int32)).cuda()
    mg = int(np.diff(gf).max()) if max_group is None else max_group
    ms = int(np.max(gs)) if max_shared is None else max_shared
    pkv().paged_attention_decode_shared(out, d["q"], d["k"], d["v"], d["bt"], d["cl"], gft, gst, mg, ms,
                                        partition_size=P)
    return out


def run_plain(batch, P=0):
    d = to_dev(batch)
    out = torch.full_like(d["q"], float("nan"))
    pkv().paged_attention_decode(out, d["q"], d["k"], d["v"], d["bt"], d["cl"], partition_size=P)
    return out


@pytest.mark.parametrize("over", [
    dict(S=16, Hq=4, Hkv=4),                              # MHA: rows = 16 sequences
    dict(S=9, Hq=16, Hkv=2, bs=32, prefix=256),           # GQA, two sequences per 16-row tile
    dict(S=7, Hq=8, Hkv=8, D=64, prefix=128, dtype="f16"),
    dict(S=20, Hq=2, Hkv=1, prefix=512),                  # group 2 > 16 rows: several tiles
])
@pytest.mark.parametrize("P", [0, 64, 512])
def test_single_group_matches_oracle(over, P):
    _single_group(over, P)


# The tcgen05 pass's own shapes: 128-row query tiles, one or two per CTA
# (groups of more than 128 rows), 128-token K/V tiles.
@pytest.mark.parametrize("over", [
    dict(S=130, Hq=2, Hkv=2, prefix=384),                 # 130 rows: a second query tile of 2 rows
    dict(S=40, Hq=8, Hkv=2, prefix=640),                  # GQA, 160 rows (4 heads x 40 sequences)
    dict(S=300, Hq=1, Hkv=1, prefix=2048),                # 300 rows: two CTAs per head, the second half full
    dict(S=140, Hq=4, Hkv=4, prefix=768, bs=256),         # a block spans two 128-token tiles
    dict(S=100, Hq=2, Hkv=2, prefix=112),                 # shared run shorter than one tile
])
@pytest.mark.parametrize("P", [0, 48, 1024])
def test_single_group_large_tiles_match_oracle(over, P):
    _single_group(over, P)


def _single_group(over, P):
    sh = synth.shrink(synth.CONFIGS["llama13b_prefix"], **over)
    b = synth.make_batch(sh, fill_unused=float("nan"))
    gf, gs = pkv().find_shared_prefix_groups(b.block_tables, b.lens, sh.bs, 4)
    assert gs.tolist() == [sh.prefix]
    out = run_shared(b, gf, gs, P)
    assert pkv().device_error() == 0
    ref = oracle_attention(b)
    assert max_err(out, ref) <= TOL[out.dtype]
    assert (out.float() - run_plain(b, P).float()).abs().max().item() <= TOL[out.dtype]


def mixed_batch(seed=3, Hq=8, Hkv=2, D=128, bs=16):
    """Seqs 0-5 share 256 tokens (A), 6-8 share nothing, 9-15 share 128 (B);
    seq 2 has no token past the shared run; seq 12 has one."""
    rng = np.random.default_rng(seed)
    S = 16
    suffix = rng.integers(1, 400, size=S)
    suffix[2] = 0
    suffix[12] = 1
    share = [256] * 6 + [0] * 3 + [128] * 7
    lens = np.array([share[s] + int(suffix[s]) for s in range(S)], dtype=np.int64)
    NB = 4000
    perm = rng.permutation(NB)
    cur = 0
    A = perm[cur:cur + 16]; cur += 16
    Bk = perm[cur:cur + 8]; cur += 8
    maxb = int((lens.max() + bs - 1) // bs) + 1
    bt = np.full((S, maxb), -1, np.int32)
    for s in range(S):
        pre = A if share[s] == 256 else (Bk if share[s] == 128 else np.array([], dtype=np.int64))
        own = -(-int(lens[s] - share[s]) // bs)
        row = np.concatenate([pre, perm[cur:cur + own]]); cur += own
        bt[s, :len(row)] = row
    g = torch.Generator().manual_seed(seed)
    k = synth.randn((NB, Hkv, bs, D), g, torch.bfloat16, "cpu")
    v = synth.randn((NB, Hkv, bs, D), g, torch.bfloat16, "cpu")
    q = synth.randn((S, Hq, D), g, torch.bfloat16, "cpu")
    sh = synth.shrink(synth.CONFIGS["llama7b"], S=S, Hq=Hq, Hkv=Hkv, D=D, bs=bs)
    return synth.Batch(sh, NB, lens, bt, perm.astype(np.int32), np.array([], np.int32), k, v, q, None, None)


@pytest.mark.parametrize("P", [0, 32, 128])
def test_mixed_groups_and_gaps(P):
    b = mixed_batch()
    gf, gs = pkv().find_shared_prefix_groups(b.block_tables, b.lens, 16, 3)
    assert gf.tolist() == [0, 6, 9, 16] and gs.tolist() == [256, 0, 128]
    out = run_shared(b, gf, gs, P)
    assert pkv().device_error() == 0
    assert max_err(out, oracle_attention(b)) <= TOL[out.dtype]


@pytest.mark.parametrize("P", [0, 32, 128])
def test_mha_mixed_groups_in_longest_first_order(P):
    """MHA, where the per-sequence kernel starts its units longest first,
    counting only a member's own tokens: members with no own token and with
    one, own lengths across several partitions, non-members and an empty
    sequence."""
    b = mixed_batch(Hq=4, Hkv=4)
    b.lens[7] = 0
    gf, gs = pkv().find_shared_prefix_groups(b.block_tables, b.lens, 16, 3)
    assert gs.tolist()[0] == 256 and gs.tolist()[-1] == 128
    out = run_shared(b, gf, gs, P)
    assert pkv().device_error() == 0
    assert torch.all(out[7].float() == 0)
    assert max_err(out, oracle_attention(b)) <= TOL[out.dtype]


def test_malformed_group_is_reported_and_falls_back():
    b = mixed_batch(seed=5)
    # 200 is not a multiple of the block size: reported, the members are then
    # attended without the prefix pass, so the output is still right.
    out = run_shared(b, [0, 6, 16], [200, 0], 0)
    assert pkv().device_error() & pkv().binding.DEVERR_CONTEXT
    assert max_err(out, oracle_attention(b)) <= TOL[out.dtype]


@pytest.mark.parametrize("P", [0, 64])
def test_group_larger_than_declared_is_reported(P):
    b = mixed_batch(seed=6)
    out = run_shared(b, [0, 6, 9, 16], [256, 0, 128], P, max_group=4)
    assert pkv().device_error() & 16
    # members past the bound are attended wholly through their own tables
    assert max_err(out, oracle_attention(b)) <= TOL[out.dtype]


@pytest.mark.parametrize("seq,entry", [(3, 7), (5, 15), (0, 2), (12, 0)])
@pytest.mark.parametrize("P", [0, 32, 128])
def test_member_whose_leading_blocks_differ_is_reported_and_uses_its_own_table(seq, entry, P):
    """Only sequences that really hold the same blocks may share the prefix
    result (openeuler.csdn.net PagedAttention explainer 6.1; aiknowledge.cn
    "2.2 PagedAttention 与 KV Cache 分页管理" 2.2.8).  One shared table entry of
    one member points at another block (holding other values): the call
    records PKV_DEVERR_GROUP and that member attends to its whole context
    through its own table, so every output still equals the oracle's.  Seq 0
    is a group's first sequence: then no other member matches it."""
    b = mixed_batch(seed=9)
    gf, gs = pkv().find_shared_prefix_groups(b.block_tables, b.lens, 16, 3)
    assert gf.tolist() == [0, 6, 9, 16] and gs.tolist() == [256, 0, 128]
    used = set(b.block_tables[b.block_tables >= 0].tolist())
    spare = next(int(x) for x in b.free_order[::-1] if int(x) not in used)
    b.block_tables[seq, entry] = spare                 # the description above no longer holds for seq
    out = run_shared(b, gf, gs, P)
    assert pkv().device_error() & pkv().binding.DEVERR_GROUP
    assert max_err(out, oracle_attention(b)) <= TOL[out.dtype]


def test_mha_tile_of_sixteen_members_with_one_stranger():
    """Multi-head attention: a prefix-pass tile holds 16 different sequences;
    the one whose leading blocks differ gets no prefix partial."""
    sh = synth.shrink(synth.CONFIGS["llama13b_prefix"], S=24, Hq=4, Hkv=4, prefix=256)
    b = synth.make_batch(sh, fill_unused=float("nan"))
    gf, gs = pkv().find_shared_prefix_groups(b.block_tables, b.lens, sh.bs, 4)
    assert gs.tolist() == [256]
    used = set(b.block_tables[b.block_tables >= 0].tolist())
    spare = next(int(x) for x in b.free_order[::-1] if int(x) not in used)
    g = torch.Generator().manual_seed(11)                # covered now: real values, not the NaN fill
    b.k_pool[spare] = synth.randn(tuple(b.k_pool[spare].shape), g, b.k_pool.dtype, "cpu")
    b.v_pool[spare] = synth.randn(tuple(b.v_pool[spare].shape), g, b.v_pool.dtype, "cpu")
    b.block_tables[10, 3] = spare
    for P in (0, 128):
        out = run_shared(b, gf, gs, P)
        assert pkv().device_error() & pkv().binding.DEVERR_GROUP
        assert max_err(out, oracle_attention(b)) <= TOL[out.dtype]


def test_session_uses_groups_for_the_prefix_workload():
    """DecodeSession finds the shared prompt and its step matches the oracle."""
    import oracle
    import paged_kv_cache_405_b200 as m
    sh = synth.shrink(synth.CONFIGS["llama13b_prefix"], S=12, Hq=4, Hkv=4)
    b = synth.make_batch(sh)
    dev = torch.device("cuda")
    k, v = b.k_pool.to(dev), b.v_pool.to(dev)
    ss = m.DecodeSession(k, v, sh.Hq, b.max_blocks, free_order=b.free_order, max_batch=sh.S)
    ss.add(-1, sh.prefix)
    prefix, _ = ss.table(-1)
    for s in range(sh.S):
        ss.add(s, int(b.lens[s]) - sh.prefix, shared_prefix=prefix, prefix_tokens=sh.prefix)
    ss.free(-1)
    plan = ss.plan(list(range(sh.S)))
    assert plan.has_groups and plan.group_shared.tolist() == [512]
    d = ss.to_device(plan)
    out = torch.empty_like(b.q, device=dev)
    ss.launch(d, b.q.to(dev), b.k_new.to(dev), b.v_new.to(dev), out)
    kc, vc = b.k_pool.clone(), b.v_pool.clone()
    oracle.kv_append(kc, vc, b.k_new, b.v_new, plan.slot_mapping)
    ref = oracle.paged_attention(b.q, kc, vc, plan.block_tables, plan.lens)
    assert m.device_error() == 0
    assert max_err(out, ref) <= TOL[out.dtype]


def test_shared_run_longer_than_declared_is_reported():
    b = mixed_batch(seed=8)
    out = run_shared(b, [0, 6, 9, 16], [256, 0, 128], 0, max_shared=128)
    assert pkv().device_error() & 16
    # the group over the bound is handled without the prefix pass: still right
    assert max_err(out, oracle_attention(b)) <= TOL[out.dtype]
