"""A decode step (kv_append + decode attention) captured once in a CUDA graph
and replayed for several steps: the host validation and launch set-up of the
C ABI run at capture time, every replay reads the step's inputs, slots,
lengths and block tables from the same device buffers, which the host
refills between replays.  Checked against the oracle after every replay,
including the shared-prefix call, whose prefix pass runs on a side stream
(captured as a fork / join)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import TOL, max_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("Hq,Hkv,shared", [(8, 8, False), (16, 2, False), (8, 8, True)])
def test_decode_step_replayed_from_a_cuda_graph(Hq, Hkv, shared):
    import paged_kv_cache_405_b200 as pkv
    S, bs, D = 6, 16, 128
    sh = synth.shrink(synth.CONFIGS["llama7b"], S=S, Hq=Hq, Hkv=Hkv, len_uniform=(100, 700), seed=Hq + shared,
                      reserve_tokens=64, prefix=64 if shared else 0)
    b = synth.make_batch(sh, device="cuda")
    k, v = b.k_pool, b.v_pool
    kc, vc = k.cpu(), v.cpu()
    alloc = pkv.BlockAllocator(b.num_blocks, bs, b.free_order)
    if shared:
        alloc.seq_add(-1)
        alloc.seq_append_slots(-1, sh.prefix)
        prefix = alloc.seq_block_table(-1)[1]
    for s in range(S):
        alloc.seq_add(s)
        if shared:
            alloc.seq_share_prefix(s, prefix, sh.prefix)
            alloc.seq_append_slots(s, int(b.lens[s]) - sh.prefix)
        else:
            alloc.seq_append_slots(s, int(b.lens[s]))
    maxB = b.max_blocks
    # static device buffers the graph reads
    q = torch.empty(S, Hq, D, dtype=torch.bfloat16, device="cuda")
    kn = torch.empty(S, Hkv, D, dtype=torch.bfloat16, device="cuda")
    vn = torch.empty_like(kn)
    slots = torch.empty(S, dtype=torch.int64, device="cuda")
    lens = torch.empty(S, dtype=torch.int32, device="cuda")
    bt = torch.empty(S, maxB, dtype=torch.int32, device="cuda")
    out = torch.empty(S, Hq, D, dtype=torch.bfloat16, device="cuda")
    if shared:
        gf = torch.tensor([0, S], dtype=torch.int32, device="cuda")
        gs = torch.tensor([sh.prefix], dtype=torch.int32, device="cuda")
        n = pkv.attention_shared_workspace_bytes(S, Hq, D, maxB * bs, 0)
    else:
        n = pkv.attention_workspace_bytes(S, Hq, D, maxB * bs, 0)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device="cuda")

    def step_calls():
        pkv.kv_append(kn, vn, k, v, slots)
        if shared:
            pkv.paged_attention_decode_shared(out, q, k, v, bt, lens, gf, gs, S, sh.prefix, workspace=ws)
        else:
            pkv.paged_attention_decode(out, q, k, v, bt, lens, workspace=ws)

    def plan(step):
        st, sl, pairs = alloc.seq_append_slots_batch(list(range(S)))
        assert st == 0 and len(pairs) == 0
        st, tables, ln = alloc.seq_block_tables_batch(list(range(S)), maxB)
        assert st == 0
        g = torch.Generator().manual_seed(100 + step)
        return (synth.randn((S, Hq, D), g, torch.bfloat16, "cpu"), synth.randn((S, Hkv, D), g, torch.bfloat16, "cpu"),
                synth.randn((S, Hkv, D), g, torch.bfloat16, "cpu"), np.asarray(sl, np.int64), tables, ln)

    def fill(p):
        qh, knh, vnh, sl, tables, ln = p
        q.copy_(qh)
        kn.copy_(knh)
        vn.copy_(vnh)
        slots.copy_(torch.from_numpy(sl))
        lens.copy_(torch.from_numpy(np.asarray(ln, np.int32)))
        bt.copy_(torch.from_numpy(np.ascontiguousarray(tables, np.int32)))

    def check(p):
        qh, knh, vnh, sl, tables, ln = p
        oracle.kv_append(kc, vc, knh, vnh, sl)
        ref = oracle.paged_attention(qh, kc, vc, tables, ln)
        assert pkv.device_error() == 0
        assert max_err(out, ref) <= TOL[out.dtype]

    p = plan(0)                     # step 0 runs eagerly (first-call set-up happens here)
    fill(p)
    step_calls()
    torch.cuda.synchronize()
    check(p)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):   # capture only: nothing runs
        step_calls()
    before = pkv.launch_count()
    for step in range(1, 4):
        p = plan(step)
        fill(p)
        graph.replay()
        torch.cuda.synchronize()
        check(p)
    assert pkv.launch_count() == before   # replays launch through the graph, not the library
    assert torch.equal(k.cpu(), kc) and torch.equal(v.cpu(), vc)
