"""DecodeSession through its host-buffer path (``step`` and ``upload``):
several decode steps with a fork (copy-on-write of the shared last block),
against the oracle allocator, ``block_copy``, ``kv_append`` and attention."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import TOL, max_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 2)])
def test_session_steps_from_host_buffers_match_oracle(Hq, Hkv):
    import paged_kv_cache_405_b200 as m
    sh = synth.shrink(synth.CONFIGS["llama7b"], S=5, Hq=Hq, Hkv=Hkv, len_uniform=(1, 300), seed=11,
                      reserve_tokens=64)
    b = synth.make_batch(sh)
    dev = torch.device("cuda")
    k, v = b.k_pool.to(dev), b.v_pool.to(dev)
    ss = m.DecodeSession(k, v, sh.Hq, b.max_blocks, free_order=b.free_order, max_batch=2 * sh.S,
                         partition_size=32)
    orc = oracle.Allocator(b.num_blocks, sh.bs, b.free_order)
    kc, vc = b.k_pool.clone(), b.v_pool.clone()
    for s in range(sh.S):
        ss.add(s, int(b.lens[s]))
        orc.seq_add(s)
        assert orc.seq_append_slots(s, int(b.lens[s]))[0] == 0
    g = torch.Generator().manual_seed(5)
    attend = list(range(sh.S))
    # a sampled continuation of a sequence whose last block is partly filled
    # at step 2 shares all its blocks, so its first write copies that block
    parent = next(s for s in range(sh.S) if (int(b.lens[s]) + 2) % sh.bs != 0)
    for step in range(5):
        if step == 2:
            ss.fork(parent, 100)
            orc.seq_fork(parent, 100)
            attend = attend + [100]
        n = len(attend)
        q = synth.randn((n, sh.Hq, sh.D), g, torch.bfloat16, "cpu").pin_memory()
        kn = synth.randn((n, sh.Hkv, sh.D), g, torch.bfloat16, "cpu").pin_memory()
        vn = synth.randn((n, sh.Hkv, sh.D), g, torch.bfloat16, "cpu").pin_memory()
        out = ss.step(q, kn, vn, attend).clone()
        slots, pairs = [], []
        for sid in attend:
            st, sl, pr = orc.seq_append_slots(sid, 1)
            assert st == 0
            slots += sl
            pairs += pr
        if step == 2:
            assert pairs, "the fork must copy the shared partial block"
        oracle.block_copy(kc, vc, pairs)
        oracle.kv_append(kc, vc, kn, vn, slots)
        bt = np.full((n, b.max_blocks), -1, np.int32)
        lens = np.zeros(n, np.int64)
        for i, sid in enumerate(attend):
            _, t, L = orc.seq_block_table(sid)
            bt[i, :len(t)] = t
            lens[i] = L
        ref = oracle.paged_attention(q, kc, vc, bt, lens)
        assert m.device_error() == 0
        assert max_err(out, ref) <= TOL[out.dtype], step
    assert torch.equal(k.cpu(), kc) and torch.equal(v.cpu(), vc)


def test_back_to_back_uploads_keep_their_plans():
    """Plans uploaded one after another without waiting (the staging buffers
    alternate and wait for their previous copy) arrive intact."""
    import paged_kv_cache_405_b200 as m
    sh = synth.shrink(synth.CONFIGS["llama7b"], S=6, Hq=4, Hkv=4, len_uniform=(1, 200), seed=12,
                      reserve_tokens=64)
    b = synth.make_batch(sh)
    dev = torch.device("cuda")
    ss = m.DecodeSession(b.k_pool.to(dev), b.v_pool.to(dev), sh.Hq, b.max_blocks, free_order=b.free_order,
                         max_batch=sh.S)
    for s in range(sh.S):
        ss.add(s, int(b.lens[s]))
    plans = [ss.plan(list(range(sh.S))) for _ in range(5)]
    devs = [ss.upload(p) for p in plans]
    torch.cuda.synchronize()
    for p, d in zip(plans, devs):
        assert np.array_equal(d.slot_mapping.cpu().numpy(), p.slot_mapping)
        assert np.array_equal(d.lens.cpu().numpy(), p.lens)
        assert np.array_equal(d.block_tables.cpu().numpy(), p.block_tables)
        assert d.cow_pairs.shape == (0, 2) and d.n_cow == 0


@pytest.mark.parametrize("prefix_tokens", [20, 33])
def test_add_with_a_prefix_ending_inside_a_block_copies_that_block(prefix_tokens):
    """Sequences mapped onto a prompt that ends part-way through a block: each
    one's first token lands in a private copy of that shared block (made by
    ``add``), the prompt's owner keeps the original; pools and attention match
    the oracle allocator + block_copy + kv_append + attention."""
    import paged_kv_cache_405_b200 as m
    NB, Hq, Hkv, bs, D, S, n_own = 24, 8, 2, 16, 64, 3, 5
    g = torch.Generator().manual_seed(prefix_tokens)
    k0 = synth.randn((NB, Hkv, bs, D), g, torch.bfloat16, "cpu")
    v0 = synth.randn((NB, Hkv, bs, D), g, torch.bfloat16, "cpu")
    order = list(np.random.default_rng(prefix_tokens).permutation(NB))
    dev = torch.device("cuda")
    k, v = k0.to(dev), v0.to(dev)
    ss = m.DecodeSession(k, v, Hq, 8, free_order=order, max_batch=S, share_prefixes=False)
    orc = oracle.Allocator(NB, bs, order)
    kc, vc = k0.clone(), v0.clone()

    def write(slots, kn, vn, pairs=()):
        oracle.block_copy(kc, vc, list(pairs))
        oracle.kv_append(kc, vc, kn, vn, slots)
        m.kv_append(kn.to(dev), vn.to(dev), k, v, torch.tensor(slots, dtype=torch.int64, device=dev))

    slots = ss.add(-1, prefix_tokens)                      # the prompt's owner
    orc.seq_add(-1)
    st, oslots, _ = orc.seq_append_slots(-1, prefix_tokens)
    assert st == 0 and oslots == slots
    write(slots, synth.randn((prefix_tokens, Hkv, D), g, torch.bfloat16, "cpu"),
          synth.randn((prefix_tokens, Hkv, D), g, torch.bfloat16, "cpu"))
    prompt, _ = ss.table(-1)
    for s in range(S):
        slots = ss.add(s, n_own, shared_prefix=prompt, prefix_tokens=prefix_tokens)
        orc.seq_add(s)
        assert orc.seq_share_prefix(s, prompt, prefix_tokens) == 0
        st, oslots, pairs = orc.seq_append_slots(s, n_own)
        assert st == 0 and oslots == slots and len(pairs) == 1      # the shared partial block is copied
        write(slots, synth.randn((n_own, Hkv, D), g, torch.bfloat16, "cpu"),
              synth.randn((n_own, Hkv, D), g, torch.bfloat16, "cpu"), pairs)
    torch.cuda.synchronize()
    assert torch.equal(k.cpu(), kc) and torch.equal(v.cpu(), vc)
    ids = [-1] + list(range(S))
    bt = np.full((len(ids), 8), -1, np.int32)
    lens = np.zeros(len(ids), np.int32)
    for i, sid in enumerate(ids):
        t, L = ss.table(sid)
        assert (t, L) == tuple(orc.seq_block_table(sid)[1:])
        bt[i, :len(t)] = t
        lens[i] = L
    q = synth.randn((len(ids), Hq, D), g, torch.bfloat16, "cpu")
    out = torch.empty(len(ids), Hq, D, dtype=torch.bfloat16, device=dev)
    m.paged_attention_decode(out, q.to(dev), k, v, torch.from_numpy(bt).to(dev), torch.from_numpy(lens).to(dev))
    ref = oracle.paged_attention(q, kc, vc, bt, lens)
    assert m.device_error() == 0
    assert max_err(out, ref) <= TOL[out.dtype]


def packed_inputs(rows, T, sh, dt, g):
    """q, new K, new V in one pinned buffer at 256-byte aligned offsets (the
    layout launch_step sends with one copy)."""
    shapes = [(rows, sh.Hq, sh.D), (T, sh.Hkv, sh.D), (T, sh.Hkv, sh.D)]
    esz = torch.empty((), dtype=dt).element_size()
    offs, total = [], 0
    for shp in shapes:
        offs.append(total)
        total += (int(np.prod(shp)) * esz + 255) // 256 * 256
    buf = torch.empty(total, dtype=torch.uint8).pin_memory()
    views = []
    for shp, o in zip(shapes, offs):
        v = buf[o:o + int(np.prod(shp)) * esz].view(dt).view(shp)
        v.copy_(synth.randn(shp, g, dt, "cpu"))
        views.append(v)
    return views


@pytest.mark.parametrize("packed", [False, True])
@pytest.mark.parametrize("cfg,over", [
    ("llama13b_prefix", dict(S=12, Hq=4, Hkv=4)),                              # shared-prefix groups
    ("longctx_beam", dict(S=2, Hq=16, Hkv=2, len_fixed=2000)),                 # forks: copy-on-write pairs
    ("spec_verify", dict(S=5, Hq=8, Hkv=2, len_uniform=(20, 700))),            # causal chunks
    ("llama7b_fp8", dict(S=6, Hq=4, Hkv=4, len_uniform=(1, 600))),             # FP8 pools
    ("llama3_gqa_bs32", dict(S=4, len_fixed=None, len_uniform=(1, 900))),      # grouped-query heads
])
def test_launch_step_planned_ahead_matches_oracle(cfg, over, packed):
    """DecodeSession.launch_step from pinned host buffers, the next step
    planned while the device works (as bench.py's end-to-end leg does),
    on every kind of plan: after each step the output equals the oracle's
    attention and, at the end, both pools equal the oracle's copies and
    appends.  Layouts repeat from step to step, so staging and device buffers
    are reused."""
    import bench
    import paged_kv_cache_405_b200 as m
    sh = synth.shrink(synth.CONFIGS[cfg], reserve_tokens=64, **over)
    dev = torch.device("cuda")
    wl = bench.Workload(sh, sh.seed, dev, 0)
    ss = wl.session
    kc, vc = ss.k_pool.cpu(), ss.v_pool.cpu()
    dt = synth.DTYPES[sh.dtype]
    g = torch.Generator().manual_seed(31)
    out_host = None
    p = wl.plan()
    for step in range(4):
        T = len(p.slot_mapping)
        rows = T if sh.chunk else len(p.seq_ids)
        if packed:           # one host buffer: one copy
            q, kn, vn = packed_inputs(rows, T, sh, dt, g)
        else:
            q = synth.randn((rows, sh.Hq, sh.D), g, dt, "cpu").pin_memory()
            kn = synth.randn((T, sh.Hkv, sh.D), g, dt, "cpu").pin_memory()
            vn = synth.randn((T, sh.Hkv, sh.D), g, dt, "cpu").pin_memory()
        done = torch.cuda.Event()
        out_host = ss.launch_step(p, q, kn, vn, out_host, out_ready=done)
        nxt = wl.plan()                          # planned while this step runs
        done.synchronize()                       # the output is on the host
        oracle.block_copy(kc, vc, p.cow_pairs)
        if sh.kv_fp8:
            oracle.kv_append_fp8(kc.numpy(), vc.numpy(), kn, vn, sh.kv_scale, sh.kv_scale, p.slot_mapping)
            ref = oracle.paged_attention_kv(q, kc.numpy(), vc.numpy(), sh.kv_scale, sh.kv_scale, p.block_tables,
                                            p.lens, threads=oracle.max_threads())
        else:
            oracle.kv_append(kc, vc, kn, vn, p.slot_mapping)
            if sh.chunk:
                ref = oracle.paged_attention_chunk(q, kc, vc, p.block_tables, p.lens, p.query_start,
                                                   threads=oracle.max_threads())
            else:
                ref = oracle.paged_attention(q, kc, vc, p.block_tables, p.lens, threads=oracle.max_threads())
        assert m.device_error() == 0
        assert max_err(out_host, ref) <= TOL[dt], step
        if cfg == "llama13b_prefix":
            assert p.has_groups
        if cfg == "longctx_beam":
            assert len(p.cow_pairs) == sh.S * (sh.beams - 1)
        p = nxt
    bits = (lambda t: t.view(torch.uint8)) if sh.kv_fp8 else (lambda t: t.view(torch.int16))
    assert torch.equal(bits(ss.k_pool.cpu()), bits(kc)) and torch.equal(bits(ss.v_pool.cpu()), bits(vc))
    assert len(ss._layouts) <= 2          # one layout per kind of step (the first may differ)


@pytest.mark.parametrize("cfg,over", [
    ("llama13b_prefix", dict(S=12, Hq=4, Hkv=4)),                              # shared-prefix groups
    ("longctx_beam", dict(S=2, Hq=16, Hkv=2, len_fixed=2000)),                 # forks: copy-on-write pairs
    ("spec_verify", dict(S=5, Hq=8, Hkv=2, len_uniform=(20, 700))),            # causal chunks
    ("llama7b_fp8", dict(S=6, Hq=4, Hkv=4, len_uniform=(1, 600))),             # FP8 pools
])
@pytest.mark.parametrize("overlap_out", [True, False])
def test_launch_step_two_in_flight_matches_oracle(cfg, over, overlap_out):
    """Two steps in flight, as bench.py's end-to-end leg runs them: step i+1
    is planned and issued before the host waits for step i's output, each
    step writing its own pinned output buffer (two alternate) and reading its
    own pinned inputs; the output copies on the session's output stream
    (waited for through launch_step's out_ready event) or on the caller's
    stream.  Every step's output equals the oracle's attention on the pools
    after that step, and at the end both pools equal the oracle's copies and
    appends."""
    import bench
    import paged_kv_cache_405_b200 as m
    sh = synth.shrink(synth.CONFIGS[cfg], reserve_tokens=64, **over)
    dev = torch.device("cuda")
    wl = bench.Workload(sh, sh.seed, dev, 0, overlap_output_copies=overlap_out)
    ss = wl.session
    kc, vc = ss.k_pool.cpu(), ss.v_pool.cpu()
    dt = synth.DTYPES[sh.dtype]
    g = torch.Generator().manual_seed(47)
    rows0 = sh.S * max(1, sh.chunk)
    outs = [torch.empty((rows0, sh.Hq, sh.D), dtype=dt).pin_memory() for _ in range(2)]
    pending = []                                 # (event, plan, q, new K, new V, out) not yet checked
    stream = torch.cuda.current_stream()

    def check(ev, p, q, kn, vn, out):
        ev.synchronize()                         # this step's output is on the host
        oracle.block_copy(kc, vc, p.cow_pairs)
        if sh.kv_fp8:
            oracle.kv_append_fp8(kc.numpy(), vc.numpy(), kn, vn, sh.kv_scale, sh.kv_scale, p.slot_mapping)
            ref = oracle.paged_attention_kv(q, kc.numpy(), vc.numpy(), sh.kv_scale, sh.kv_scale, p.block_tables,
                                            p.lens, threads=oracle.max_threads())
        else:
            oracle.kv_append(kc, vc, kn, vn, p.slot_mapping)
            if sh.chunk:
                ref = oracle.paged_attention_chunk(q, kc, vc, p.block_tables, p.lens, p.query_start,
                                                   threads=oracle.max_threads())
            else:
                ref = oracle.paged_attention(q, kc, vc, p.block_tables, p.lens, threads=oracle.max_threads())
        assert max_err(out, ref) <= TOL[dt]

    p = wl.plan()
    for step in range(5):
        T = len(p.slot_mapping)
        rows = T if sh.chunk else len(p.seq_ids)
        q, kn, vn = packed_inputs(rows, T, sh, dt, g)
        ev = torch.cuda.Event()
        outs[step % 2] = ss.launch_step(p, q, kn, vn, outs[step % 2], stream=stream, out_ready=ev)
        pending.append((ev, p, q, kn, vn, outs[step % 2]))
        p = wl.plan()                            # the step after, planned while two are in flight
        if len(pending) == 2:
            check(*pending.pop(0))
    for item in pending:
        check(*item)
    assert m.device_error() == 0
    bits = (lambda t: t.view(torch.uint8)) if sh.kv_fp8 else (lambda t: t.view(torch.int16))
    assert torch.equal(bits(ss.k_pool.cpu()), bits(kc)) and torch.equal(bits(ss.v_pool.cpu()), bits(vc))
