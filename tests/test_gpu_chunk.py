"""GPU parity of the causal chunk path (pkv_paged_attention_chunk) against the
oracle: several new tokens per sequence, each attending to the cache up to and
including its own position."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import TOL, max_err, to_dev

pytestmark = pytest.mark.gpu


def chunk_case(Hq, Hkv, D, bs, dtype, seed, S=7, max_n=8, lens=None, ns=None):
    sh = synth.shrink(synth.CONFIGS["llama7b"], S=S, Hq=Hq, Hkv=Hkv, D=D, bs=bs, dtype=dtype, seed=seed,
                      len_uniform=(1, 700) if lens is None else None, lens=lens)
    b = synth.make_batch(sh, fill_unused=float("nan"))
    rng = np.random.default_rng(seed)
    if ns is None:
        ns = [int(rng.integers(1, min(max_n, int(L)) + 1)) if L > 0 else 0 for L in b.lens]
    qs = np.concatenate([[0], np.cumsum(ns)]).astype(np.int32)
    T = int(qs[-1])
    g = torch.Generator().manual_seed(seed + 99)
    q = synth.randn((T, Hq, D), g, synth.DTYPES[dtype], "cpu")
    return b, q, qs, max(ns)


def run_chunk(b, q, qs, max_n, P):
    import paged_kv_cache_405_b200 as pkv
    d = to_dev(b)
    out = torch.full((q.shape[0],) + tuple(q.shape[1:]), float("nan"), dtype=q.dtype, device="cuda")
    pkv.paged_attention_chunk(out, q.cuda(), d["k"], d["v"], d["bt"], d["cl"], torch.from_numpy(qs).cuda(), max_n,
                              partition_size=P)
    return out


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 2), (16, 2), (32, 2), (4, 1)])
@pytest.mark.parametrize("bs,D", [(16, 128), (32, 64), (64, 128)])
@pytest.mark.parametrize("P", [0, 32, 128])
def test_chunk_matches_oracle(dtype, Hq, Hkv, bs, D, P):
    import paged_kv_cache_405_b200 as pkv
    b, q, qs, max_n = chunk_case(Hq, Hkv, D, bs, dtype, seed=Hq * 13 + bs + D + P)
    out = run_chunk(b, q, qs, max_n, P)
    assert pkv.device_error() == 0
    ref = oracle.paged_attention_chunk(q, b.k_pool, b.v_pool, b.block_tables, b.lens, qs,
                                       threads=oracle.max_threads())
    assert max_err(out, ref) <= TOL[out.dtype]


@pytest.mark.parametrize("P", [0, 16, 64])
def test_whole_prompt_and_edge_chunks(P):
    """A chunk equal to the whole context (prefill from empty), one-token
    chunks, chunks ending exactly on block and partition boundaries."""
    import paged_kv_cache_405_b200 as pkv
    lens = [1, 16, 17, 64, 65, 300, 512, 40]
    ns = [1, 16, 17, 3, 64, 16, 9, 40]
    b, q, qs, max_n = chunk_case(8, 2, 128, 16, "bf16", seed=5, S=len(lens), lens=lens, ns=ns)
    out = run_chunk(b, q, qs, max_n, P)
    assert pkv.device_error() == 0
    ref = oracle.paged_attention_chunk(q, b.k_pool, b.v_pool, b.block_tables, b.lens, qs,
                                       threads=oracle.max_threads())
    assert max_err(out, ref) <= TOL[out.dtype]


def test_one_token_chunks_equal_decode():
    import paged_kv_cache_405_b200 as pkv
    sh = synth.shrink(synth.CONFIGS["llama3_gqa_bs16"], S=6, len_fixed=None, len_uniform=(1, 900))
    b = synth.make_batch(sh)
    d = to_dev(b)
    qs = torch.arange(sh.S + 1, dtype=torch.int32, device="cuda")
    a = torch.empty_like(d["q"])
    pkv.paged_attention_chunk(a, d["q"], d["k"], d["v"], d["bt"], d["cl"], qs, 1)
    c = torch.empty_like(d["q"])
    pkv.paged_attention_decode(c, d["q"], d["k"], d["v"], d["bt"], d["cl"])
    assert pkv.device_error() == 0
    assert (a.float() - c.float()).abs().max().item() <= TOL[a.dtype]


def test_bad_query_start_is_reported():
    import paged_kv_cache_405_b200 as pkv
    b, q, qs, max_n = chunk_case(8, 8, 128, 16, "bf16", seed=3, S=3, lens=[10, 20, 30], ns=[2, 2, 2])
    bad = qs.copy()
    bad[2] = 99                      # beyond num_tokens
    out = run_chunk(b, q, bad, max_n, 0)
    assert pkv.device_error() & pkv.binding.DEVERR_CONTEXT
    del out


def test_session_chunk_step_matches_oracle():
    """DecodeSession: reserve 3 draft tokens per sequence, write their K/V,
    attend causally; the oracle replays the same writes on the CPU."""
    import paged_kv_cache_405_b200 as m
    sh = synth.shrink(synth.CONFIGS["spec_verify"], S=5, len_uniform=(20, 700), chunk=3)
    b = synth.make_batch(sh)
    dev = torch.device("cuda")
    k, v = b.k_pool.to(dev), b.v_pool.to(dev)
    ss = m.DecodeSession(k, v, sh.Hq, b.max_blocks, free_order=b.free_order, max_batch=sh.S)
    for s in range(sh.S):
        ss.add(s, int(b.lens[s]))
    ss.reserve_chunk_workspace(sh.S * sh.chunk)
    plan = ss.plan_chunk(list(range(sh.S)), [sh.chunk] * sh.S)
    T = sh.S * sh.chunk
    g = torch.Generator().manual_seed(11)
    q = synth.randn((T, sh.Hq, sh.D), g, torch.bfloat16, "cpu")
    kn = synth.randn((T, sh.Hkv, sh.D), g, torch.bfloat16, "cpu")
    vn = synth.randn((T, sh.Hkv, sh.D), g, torch.bfloat16, "cpu")
    out = torch.empty((T, sh.Hq, sh.D), dtype=torch.bfloat16, device=dev)
    ss.launch_chunk(ss.chunk_to_device(plan), q.to(dev), kn.to(dev), vn.to(dev), out)
    kc, vc = b.k_pool.clone(), b.v_pool.clone()
    oracle.kv_append(kc, vc, kn, vn, plan.slot_mapping)
    ref = oracle.paged_attention_chunk(q, kc, vc, plan.block_tables, plan.lens, plan.query_start,
                                       threads=oracle.max_threads())
    assert m.device_error() == 0
    assert torch.equal(k.cpu(), kc) and torch.equal(v.cpu(), vc)
    assert max_err(out, ref) <= TOL[out.dtype]
