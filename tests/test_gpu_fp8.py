"""GPU parity of the FP8 E4M3 pools: quantizing append byte for byte, decode
attention element by element, against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import TOL, max_err

pytestmark = pytest.mark.gpu


def fp8_pools(b, seed, k_scale, v_scale):
    """E4M3 code pools: N(0,1) values / scale cast by torch's float8_e4m3fn;
    rows no context covers hold the NaN code."""
    g = torch.Generator().manual_seed(seed)
    shape = tuple(b.k_pool.shape)
    kc = (torch.randn(shape, generator=g) / k_scale).to(torch.float8_e4m3fn).view(torch.uint8)
    vc = (torch.randn(shape, generator=g) / v_scale).to(torch.float8_e4m3fn).view(torch.uint8)
    covered = torch.zeros(shape[0], shape[2], dtype=torch.bool)
    bs = shape[2]
    for s in range(b.shape.S):
        L = int(b.lens[s])
        for j in range(-(-L // bs)):
            covered[int(b.block_tables[s, j]), : min(bs, L - j * bs)] = True
    mask = ~covered[:, None, :, None].expand(shape)
    kc[mask] = 0x7F
    vc[mask] = 0x7F
    return kc.contiguous(), vc.contiguous()


@pytest.mark.parametrize("src", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("scales", [(1.0, 1.0), (0.37, 2.5), (1 / 64, 1 / 16)])
def test_kv_append_fp8_bit_exact(src, scales):
    import paged_kv_cache_405_b200 as pkv
    ks, vs = scales
    NB, Hkv, bs, D, T = 40, 4, 16, 128, 23
    g = torch.Generator().manual_seed(7)
    kn = (torch.randn(T, Hkv, D, generator=g) * 30).to(src)     # some values saturate
    vn = (torch.randn(T, Hkv, D, generator=g) * 3).to(src)
    kn[0, 0, :4] = torch.tensor([0.0, -0.0, 1e-7, -1e-7]).to(src)
    slots = np.random.default_rng(1).choice(NB * bs, size=T, replace=False).astype(np.int64)
    slots[::6] = -1
    kc = np.zeros((NB, Hkv, bs, D), np.uint8)
    vc = np.zeros((NB, Hkv, bs, D), np.uint8)
    oracle.kv_append_fp8(kc, vc, kn, vn, ks, vs, slots)
    kd = torch.zeros((NB, Hkv, bs, D), dtype=torch.uint8, device="cuda")
    vd = torch.zeros_like(kd)
    pkv.kv_append_fp8(kn.cuda(), vn.cuda(), kd, vd, torch.from_numpy(slots).cuda(), ks, vs)
    assert pkv.device_error() == 0
    assert np.array_equal(kd.cpu().numpy(), kc) and np.array_equal(vd.cpu().numpy(), vc)


@pytest.mark.parametrize("src", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("scale", [1.0, 1 / 64])
def test_kv_append_fp8_rounds_ties_to_even(src, scale):
    """Every midpoint between adjacent E4M3 values, as an exact tie after the
    x * (1/scale) product (power-of-two scales), quantized bit-exactly like
    the oracle (ties to the even code)."""
    import paged_kv_cache_405_b200 as pkv
    from test_oracle_pins import e4m3_midpoints
    NB, Hkv, bs, D, T = 4, 2, 16, 128, 2
    mids = e4m3_midpoints() * scale
    flat = torch.zeros(T * Hkv * D)
    flat[:len(mids)] = mids
    kn = flat.view(T, Hkv, D).to(src)
    assert torch.equal(kn.float(), flat.view(T, Hkv, D))      # the ties are exact in the input type
    vn = kn.flip(0)
    slots = np.array([5, 37], np.int64)
    kc = np.zeros((NB, Hkv, bs, D), np.uint8)
    vc = np.zeros((NB, Hkv, bs, D), np.uint8)
    oracle.kv_append_fp8(kc, vc, kn, vn, scale, scale, slots)
    kd = torch.zeros((NB, Hkv, bs, D), dtype=torch.uint8, device="cuda")
    vd = torch.zeros_like(kd)
    pkv.kv_append_fp8(kn.cuda(), vn.cuda(), kd, vd, torch.from_numpy(slots).cuda(), scale, scale)
    assert pkv.device_error() == 0
    assert np.array_equal(kd.cpu().numpy(), kc) and np.array_equal(vd.cpu().numpy(), vc)


@pytest.mark.parametrize("qdt", ["bf16", "f16"])
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 2), (8, 1), (32, 2), (40, 2)])
@pytest.mark.parametrize("bs,D", [(16, 128), (64, 128), (32, 64)])
@pytest.mark.parametrize("P", [0, 32, 512])
def test_decode_fp8_matches_oracle(qdt, Hq, Hkv, bs, D, P):
    import paged_kv_cache_405_b200 as pkv
    sh = synth.shrink(synth.CONFIGS["llama7b"], S=6, Hq=Hq, Hkv=Hkv, bs=bs, D=D, dtype=qdt,
                      len_uniform=(1, 900), seed=Hq + bs + D + P)
    b = synth.make_batch(sh)
    ks, vs = 1 / 32, 1 / 8
    kc, vc = fp8_pools(b, 5, ks, vs)
    ref = oracle.paged_attention_kv(b.q, kc, vc, ks, vs, b.block_tables, b.lens, threads=oracle.max_threads())
    out = torch.full_like(b.q, float("nan"), device="cuda")
    pkv.paged_attention_decode_fp8(out, b.q.cuda(), kc.cuda(), vc.cuda(), torch.from_numpy(b.block_tables).cuda(),
                                   torch.from_numpy(b.lens.astype(np.int32)).cuda(), ks, vs, partition_size=P)
    assert pkv.device_error() == 0
    assert max_err(out, ref) <= TOL[out.dtype]


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 4)])
def test_decode_fp8_empty_and_one_token_contexts(Hq, Hkv):
    """Zero-length contexts give zeros; one-token contexts give that token's
    value (dequantized), through both the per-head and the grouped kernel."""
    import paged_kv_cache_405_b200 as pkv
    sh = synth.shrink(synth.CONFIGS["llama7b"], S=7, Hq=Hq, Hkv=Hkv, len_uniform=(1, 40), seed=3)
    b = synth.make_batch(sh)
    lens = b.lens.copy()
    lens[[0, 3]] = 0
    lens[[1, 5]] = 1
    ks, vs = 1 / 16, 1 / 4
    kc, vc = fp8_pools(b, 2, ks, vs)
    ref = oracle.paged_attention_kv(b.q, kc, vc, ks, vs, b.block_tables, lens, threads=oracle.max_threads())
    out = torch.full_like(b.q, float("nan"), device="cuda")
    pkv.paged_attention_decode_fp8(out, b.q.cuda(), kc.cuda(), vc.cuda(), torch.from_numpy(b.block_tables).cuda(),
                                   torch.from_numpy(lens.astype(np.int32)).cuda(), ks, vs)
    assert pkv.device_error() == 0
    o = out.float().cpu()
    assert torch.all(o[[0, 3]] == 0)
    assert max_err(out, ref) <= TOL[out.dtype]


@pytest.mark.parametrize("S,P", [(9, 32), (100, 64), (144, 128), (256, 32), (300, 32)])
def test_decode_fp8_unit_order_edge_lengths(S, P):
    """Contexts at and around multiples of the partition (0, 1, P-1, P, P+1,
    2P, ...) over batches whose longest-first unit order the per-head kernel
    derives with one, four and eight sequences per lane (S up to 256 and at
    most 1024 sequences x partitions), and past those bounds (grid order):
    every unit is attended exactly once."""
    import paged_kv_cache_405_b200 as pkv
    rng = np.random.default_rng(S + P)
    edge = [0, 1, P - 1, P, P + 1, 2 * P, 2 * P + 15, 3 * P - 1, 5 * P]
    lens = [edge[i] if i < len(edge) else int(rng.integers(0, 5 * P + 1)) for i in range(S)]
    rng.shuffle(lens)
    sh = synth.shrink(synth.CONFIGS["llama7b"], S=S, Hq=2, Hkv=2, lens=lens, len_uniform=None, seed=S)
    b = synth.make_batch(sh)
    ks, vs = 1 / 32, 1 / 8
    kc, vc = fp8_pools(b, 6, ks, vs)
    ref = oracle.paged_attention_kv(b.q, kc, vc, ks, vs, b.block_tables, b.lens, threads=oracle.max_threads())
    out = torch.full_like(b.q, float("nan"), device="cuda")
    pkv.paged_attention_decode_fp8(out, b.q.cuda(), kc.cuda(), vc.cuda(), torch.from_numpy(b.block_tables).cuda(),
                                   torch.from_numpy(b.lens.astype(np.int32)).cuda(), ks, vs, partition_size=P)
    assert pkv.device_error() == 0
    assert torch.all(out.float().cpu()[torch.from_numpy(b.lens == 0)] == 0)
    assert max_err(out, ref) <= TOL[out.dtype]


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 4)])
def test_decode_fp8_query_magnitudes(Hq, Hkv):
    """Query rows spanning many orders of magnitude (down into the FP16
    subnormal range the query is rounded to), a zero head and an all-zero
    sequence."""
    import paged_kv_cache_405_b200 as pkv
    sh = synth.shrink(synth.CONFIGS["llama7b"], S=6, Hq=Hq, Hkv=Hkv, len_uniform=(1, 400), seed=8)
    b = synth.make_batch(sh)
    q = b.q.float().clone()
    for s, f in enumerate([1e-4, 3e-2, 1.0, 2.5, 6.0, 0.0]):
        q[s] *= f
    q[2, 0] = 0.0                       # one zero head inside an otherwise ordinary sequence
    q = q.to(b.q.dtype)
    ks, vs = 1 / 16, 1 / 4
    kc, vc = fp8_pools(b, 4, ks, vs)
    ref = oracle.paged_attention_kv(q, kc, vc, ks, vs, b.block_tables, b.lens, threads=oracle.max_threads())
    out = torch.full_like(q, float("nan"), device="cuda")
    pkv.paged_attention_decode_fp8(out, q.cuda(), kc.cuda(), vc.cuda(), torch.from_numpy(b.block_tables).cuda(),
                                   torch.from_numpy(b.lens.astype(np.int32)).cuda(), ks, vs)
    assert pkv.device_error() == 0
    assert max_err(out, ref) <= TOL[out.dtype]


def test_fp8_decode_step_end_to_end():
    """Quantized append of one new token per sequence, then attention over
    L+1 tokens, against the oracle's quantizer and attention."""
    import paged_kv_cache_405_b200 as pkv
    sh = synth.shrink(synth.CONFIGS["llama3_gqa_bs16"], S=5, len_fixed=None, len_uniform=(1, 600))
    b = synth.make_batch(sh)
    ks, vs = 0.05, 0.2
    kc, vc = fp8_pools(b, 9, ks, vs)
    slots = np.array([int(b.block_tables[s, int(b.lens[s]) // sh.bs]) * sh.bs + int(b.lens[s]) % sh.bs
                      if int(b.lens[s]) // sh.bs < b.max_blocks and b.block_tables[s, int(b.lens[s]) // sh.bs] >= 0
                      else -1 for s in range(sh.S)], np.int64)
    lens = b.lens + (slots >= 0)
    kcn, vcn = kc.numpy().copy(), vc.numpy().copy()
    oracle.kv_append_fp8(kcn, vcn, b.k_new, b.v_new, ks, vs, slots)
    ref = oracle.paged_attention_kv(b.q, kcn, vcn, ks, vs, b.block_tables, lens, threads=oracle.max_threads())
    kd, vd = kc.cuda(), vc.cuda()
    pkv.kv_append_fp8(b.k_new.cuda(), b.v_new.cuda(), kd, vd, torch.from_numpy(slots).cuda(), ks, vs)
    out = torch.empty_like(b.q, device="cuda")
    pkv.paged_attention_decode_fp8(out, b.q.cuda(), kd, vd, torch.from_numpy(b.block_tables).cuda(),
                                   torch.from_numpy(lens.astype(np.int32)).cuda(), ks, vs)
    assert pkv.device_error() == 0
    assert np.array_equal(kd.cpu().numpy(), kcn) and np.array_equal(vd.cpu().numpy(), vcn)
    assert max_err(out, ref) <= TOL[out.dtype]


def test_session_fp8_step_matches_oracle():
    import paged_kv_cache_405_b200 as m
    sh = synth.shrink(synth.CONFIGS["llama7b_fp8"], S=5, Hq=8, Hkv=8, len_uniform=(1, 500))
    b = synth.make_batch(sh)
    dev = torch.device("cuda")
    k, v = b.k_pool.to(dev), b.v_pool.to(dev)
    ss = m.DecodeSession(k, v, sh.Hq, b.max_blocks, free_order=b.free_order, max_batch=sh.S,
                         kv_scales=(sh.kv_scale, sh.kv_scale))
    for s in range(sh.S):
        ss.add(s, int(b.lens[s]))
    plan = ss.plan(list(range(sh.S)))
    out = torch.empty_like(b.q, device=dev)
    ss.launch(ss.to_device(plan), b.q.to(dev), b.k_new.to(dev), b.v_new.to(dev), out)
    kc, vc = b.k_pool.numpy().copy(), b.v_pool.numpy().copy()
    oracle.kv_append_fp8(kc, vc, b.k_new, b.v_new, sh.kv_scale, sh.kv_scale, plan.slot_mapping)
    ref = oracle.paged_attention_kv(b.q, kc, vc, sh.kv_scale, sh.kv_scale, plan.block_tables, plan.lens,
                                    threads=oracle.max_threads())
    assert m.device_error() == 0
    assert np.array_equal(k.cpu().numpy(), kc) and np.array_equal(v.cpu().numpy(), vc)
    assert max_err(out, ref) <= TOL[out.dtype]


def _fp8_split_case(S, Hq, lens_range, seed):
    sh = synth.shrink(synth.CONFIGS["llama7b"], S=S, Hq=Hq, Hkv=Hq, len_uniform=lens_range, seed=seed,
                      reserve_tokens=64)
    b = synth.make_batch(sh)
    ks, vs = 1 / 32, 1 / 8
    kc, vc = fp8_pools(b, seed, ks, vs)
    return b, kc, vc, ks, vs


def test_decode_fp8_in_kernel_merge_over_stale_workspace_and_repeated_calls():
    """The per-head kernel merges a row's split-K partials itself (2 to 32
    partitions of at least 512 tokens), counting arrivals in workspace words
    stamped per call: a workspace of random bytes, then of 0xff bytes, then
    back-to-back calls on the same workspace all match the oracle."""
    import paged_kv_cache_405_b200 as pkv
    P = 512
    b, kc, vc, ks, vs = _fp8_split_case(9, 4, (1, 3000), 21)
    maxB = b.block_tables.shape[1]
    assert 1 < -(-maxB * 16 // P) <= 32
    ref = oracle.paged_attention_kv(b.q, kc, vc, ks, vs, b.block_tables, b.lens, threads=oracle.max_threads())
    n = pkv.attention_workspace_bytes(b.shape.S, b.shape.Hq, 128, maxB * 16, P)
    g = torch.Generator().manual_seed(3)
    ws = torch.randint(0, 256, (n,), dtype=torch.uint8, generator=g).cuda()
    args = (b.q.cuda(), kc.cuda(), vc.cuda(), torch.from_numpy(b.block_tables).cuda(),
            torch.from_numpy(b.lens.astype(np.int32)).cuda(), ks, vs)
    for fill in ("random", "ones", "previous", "previous"):
        if fill == "ones":
            ws.fill_(0xFF)
        out = torch.full_like(b.q, float("nan"), device="cuda")
        pkv.paged_attention_decode_fp8(out, *args, partition_size=P, workspace=ws)
        assert pkv.device_error() == 0
        assert max_err(out, ref) <= TOL[out.dtype], fill


def test_decode_fp8_in_kernel_merge_replayed_from_a_cuda_graph():
    """CUDA-graph replays reuse one call stamp: every replay starts its
    arrival counts from zero (the completing arrival resets them), also when
    the lengths, and with them the partitions per row, change between
    replays."""
    import paged_kv_cache_405_b200 as pkv
    P = 512
    b, kc, vc, ks, vs = _fp8_split_case(6, 8, (600, 3000), 22)
    S, Hq, D = b.shape.S, b.shape.Hq, 128
    maxB = b.block_tables.shape[1]
    n = pkv.attention_workspace_bytes(S, Hq, D, maxB * 16, P)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    q = torch.empty(S, Hq, D, dtype=b.q.dtype, device="cuda")
    lens = torch.empty(S, dtype=torch.int32, device="cuda")
    out = torch.empty(S, Hq, D, dtype=b.q.dtype, device="cuda")
    kd, vd, bt = kc.cuda(), vc.cuda(), torch.from_numpy(b.block_tables).cuda()
    rng = np.random.default_rng(5)

    def case(step):
        g = torch.Generator().manual_seed(50 + step)
        ln = np.minimum(b.lens, rng.integers(1, 3001, size=S)).astype(np.int32)  # within each table
        ln[step % S] = 0 if step == 2 else ln[step % S]                           # an empty row once
        return synth.randn((S, Hq, D), g, b.q.dtype, "cpu"), ln

    def run():
        pkv.paged_attention_decode_fp8(out, q, kd, vd, bt, lens, ks, vs, partition_size=P, workspace=ws)

    qh, ln = case(0)
    q.copy_(qh)
    lens.copy_(torch.from_numpy(ln))
    run()                            # eager first call
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run()
    for step in range(1, 5):
        qh, ln = case(step)
        q.copy_(qh)
        lens.copy_(torch.from_numpy(ln))
        graph.replay()
        torch.cuda.synchronize()
        ref = oracle.paged_attention_kv(qh, kc, vc, ks, vs, b.block_tables, ln, threads=oracle.max_threads())
        assert pkv.device_error() == 0
        assert max_err(out, ref) <= TOL[out.dtype], step


@pytest.mark.parametrize("P,lens", [(512, (16500, 17000)), (256, (500, 3000))])
def test_decode_fp8_long_or_short_partitions_use_the_reduce(P, lens):
    """Past 32 partitions per row, or with partitions under 512 tokens, the
    per-head kernel leaves the merge to the reduce kernel; the result is the
    same."""
    import paged_kv_cache_405_b200 as pkv
    b, kc, vc, ks, vs = _fp8_split_case(3, 2, lens, 23)
    assert -(-b.block_tables.shape[1] * 16 // P) > (32 if P >= 512 else 1)
    ref = oracle.paged_attention_kv(b.q, kc, vc, ks, vs, b.block_tables, b.lens, threads=oracle.max_threads())
    out = torch.full_like(b.q, float("nan"), device="cuda")
    pkv.paged_attention_decode_fp8(out, b.q.cuda(), kc.cuda(), vc.cuda(), torch.from_numpy(b.block_tables).cuda(),
                                   torch.from_numpy(b.lens.astype(np.int32)).cuda(), ks, vs, partition_size=P)
    assert pkv.device_error() == 0
    assert max_err(out, ref) <= TOL[out.dtype]
