"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

kv_append and block_copy are compared byte for byte; attention element by
element within the tolerance in gpu_helpers.TOL.  Inputs are the seeded
synthetic batches of ``synth``, shrunk so the oracle finishes in seconds while
still spanning several tiles, partitions and a ragged tail.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import TOL, gpu_attention, max_err, oracle_attention, to_dev

pytestmark = pytest.mark.gpu


def pkv():
    import paged_kv_cache_405_b200 as m
    return m


DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


# ------------------------------------------------------------------ byte ops
@pytest.mark.parametrize("cfg,dtype", [("tiny", "f32"), ("llama7b", "bf16"), ("llama7b", "f16"),
                                       ("longctx_beam", "bf16")])
def test_kv_append_bit_exact(cfg, dtype):
    sh = synth.shrink(synth.CONFIGS[cfg], dtype=dtype, S=min(synth.CONFIGS[cfg].S, 24),
                      lens=None if cfg != "tiny" else synth.CONFIGS[cfg].lens,
                      len_fixed=None, len_uniform=(1, 300) if cfg != "tiny" else None,
                      num_blocks=None if cfg != "tiny" else 32, reserve_tokens=64)
    b = synth.make_batch(sh)
    T = sh.S
    rng = np.random.default_rng(3)
    slots = rng.choice(b.num_blocks * sh.bs, size=T, replace=False).astype(np.int64)
    slots[::5] = -1                                         # skipped tokens
    kc, vc = b.k_pool.clone(), b.v_pool.clone()
    oracle.kv_append(kc, vc, b.k_new, b.v_new, slots)
    d = to_dev(b)
    pkv().kv_append(b.k_new.cuda(), b.v_new.cuda(), d["k"], d["v"], torch.from_numpy(slots).cuda())
    assert pkv().device_error() == 0
    ki = torch.int16 if dtype != "f32" else torch.int32
    assert torch.equal(d["k"].cpu().view(ki), kc.view(ki))
    assert torch.equal(d["v"].cpu().view(ki), vc.view(ki))


@pytest.mark.parametrize("cfg", ["tiny", "llama3_gqa_bs32", "longctx_beam"])
def test_block_copy_bit_exact(cfg):
    sh = synth.shrink(synth.CONFIGS[cfg], S=4, len_fixed=None, len_uniform=(1, 200),
                      lens=None if cfg != "tiny" else [35, 16, 1, 50])
    b = synth.make_batch(sh)
    rng = np.random.default_rng(9)
    ids = rng.permutation(b.num_blocks)[:10]
    pairs = np.stack([ids[:5], ids[5:]], 1).astype(np.int32)
    kc, vc = b.k_pool.clone(), b.v_pool.clone()
    oracle.block_copy(kc, vc, pairs)
    d = to_dev(b)
    pkv().block_copy(d["k"], d["v"], torch.from_numpy(pairs).cuda())
    assert pkv().device_error() == 0
    ki = torch.int16 if b.k_pool.dtype != torch.float32 else torch.int32
    assert torch.equal(d["k"].cpu().view(ki), kc.view(ki))
    assert torch.equal(d["v"].cpu().view(ki), vc.view(ki))


# ------------------------------------------------------------------ attention
SMALL = {
    # config, overrides
    "tiny": dict(),
    "llama7b": dict(S=12, Hq=8, Hkv=8, len_uniform=(1, 700)),
    "llama13b_prefix": dict(S=16, Hq=4, Hkv=4),
    "llama3_gqa_bs16": dict(S=6, len_fixed=None, len_uniform=(1, 1100)),
    "llama3_gqa_bs32": dict(S=6, len_fixed=None, len_uniform=(1, 1100)),
    "longctx_beam": dict(S=2, Hq=16, Hkv=2, len_fixed=None, len_uniform=(3000, 5000)),
}


@pytest.mark.parametrize("cfg", list(SMALL))
@pytest.mark.parametrize("partition_size", [0, 64, 512])
def test_attention_matches_oracle(cfg, partition_size):
    sh = synth.shrink(synth.CONFIGS[cfg], **SMALL[cfg])
    b = synth.make_batch(sh, fill_unused=float("nan"))
    ref = oracle_attention(b)
    out = gpu_attention(b, partition_size=partition_size)
    assert max_err(out, ref) <= TOL[out.dtype]


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 2)])
@pytest.mark.parametrize("partition_size", [0, 128])
def test_values_scaled_by_inverse_sqrt_head_dim(dtype, Hq, Hkv, partition_size):
    """The other reading of the Llama-2-7B-shaped workload's "q/K/V ~N(0,1)
    scaled 1/sqrt(128)": the values themselves scaled, so the logits are
    ~N(0, 1/128^2) and the softmax is almost uniform over up to 2048 tokens
    (long sums of nearly equal weights instead of a peaked softmax).  The
    outputs are then ~0.09/sqrt(L), below the absolute tolerance, so they are
    also held to 2e-2 of their own largest magnitude (an all-zero output
    fails that)."""
    import math
    sh = synth.shrink(synth.CONFIGS["llama7b"], S=10, Hq=Hq, Hkv=Hkv, dtype=dtype, seed=21)
    b = synth.make_batch(sh, value_scale=1 / math.sqrt(128), fill_unused=float("nan"))
    ref = oracle_attention(b)
    out = gpu_attention(b, partition_size=partition_size)
    err = max_err(out, ref)
    assert err <= TOL[out.dtype]
    assert err <= 2e-2 * float(np.abs(ref).max())


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 4), (16, 2), (32, 2), (8, 1)])
@pytest.mark.parametrize("bs", [16, 32, 64])
@pytest.mark.parametrize("D", [64, 128])
def test_attention_shapes(dtype, Hq, Hkv, bs, D):
    sh = synth.shrink(synth.CONFIGS["llama7b"], S=5, Hq=Hq, Hkv=Hkv, bs=bs, D=D, dtype=dtype,
                      len_uniform=(1, 300), seed=Hq * 7 + bs + D)
    b = synth.make_batch(sh, fill_unused=float("nan"))
    ref = oracle_attention(b)
    for P in (0, 32):
        out = gpu_attention(b, partition_size=P)
        assert max_err(out, ref) <= TOL[out.dtype], (P,)


EDGE_LENS = [0, 1, 15, 16, 17, 63, 64, 65, 511, 512, 513, 1024]


@pytest.mark.parametrize("Hq,Hkv,dtype", [(4, 4, "bf16"), (16, 2, "bf16"), (4, 4, "f32"), (8, 1, "f16")])
@pytest.mark.parametrize("partition_size", [0, 512, 16])
def test_edge_lengths(Hq, Hkv, dtype, partition_size):
    sh = synth.shrink(synth.CONFIGS["llama7b"], S=len(EDGE_LENS), Hq=Hq, Hkv=Hkv, dtype=dtype,
                      lens=EDGE_LENS, len_uniform=None, seed=17)
    b = synth.make_batch(sh, fill_unused=float("nan"))
    ref = oracle_attention(b)
    out = gpu_attention(b, partition_size=partition_size)
    assert max_err(out, ref) <= TOL[out.dtype]
    assert torch.count_nonzero(out[0]).item() == 0          # empty context -> zeros


def test_context_fills_the_whole_table():
    """A context of exactly max_blocks_per_seq * block_size tokens."""
    sh = synth.shrink(synth.CONFIGS["llama3_gqa_bs16"], S=3, len_fixed=None, lens=[800, 800, 33])
    b = synth.make_batch(sh)
    nb = 50                                                  # 800 / 16
    bt = np.ascontiguousarray(b.block_tables[:, :nb])
    ref = oracle_attention(b, bt=bt)
    for P in (0, 128):
        out = gpu_attention(b, bt=bt, partition_size=P)
        assert max_err(out, ref) <= TOL[out.dtype]


def test_deterministic_and_split_consistent():
    sh = synth.shrink(synth.CONFIGS["longctx_beam"], S=2, Hq=16, Hkv=2, len_fixed=None, len_uniform=(2000, 4000))
    b = synth.make_batch(sh)
    d = to_dev(b)
    a1 = gpu_attention(b, partition_size=512, dev_tensors=d)
    a2 = gpu_attention(b, partition_size=512, dev_tensors=d)
    assert torch.equal(a1.view(torch.int16), a2.view(torch.int16))
    single = gpu_attention(b, partition_size=8192, dev_tensors=d)
    ref = oracle_attention(b)
    for o in (a1, single):
        assert max_err(o, ref) <= TOL[o.dtype]
    assert (a1.float() - single.float()).abs().max().item() <= TOL[a1.dtype]


def test_prefix_once_equals_copied_bit_identical():
    """A shared prefix read through shared blocks and the same prefix copied per
    sequence give bit-identical outputs (openeuler.csdn.net explainer 6.1)."""
    sh = synth.shrink(synth.CONFIGS["llama13b_prefix"], S=8, Hq=4, Hkv=4, reserve_tokens=0)
    b = synth.make_batch(sh)
    nbp = 32
    extra = sh.S * nbp
    k = torch.cat([b.k_pool, torch.zeros((extra,) + tuple(b.k_pool.shape[1:]), dtype=b.k_pool.dtype)])
    v = torch.cat([b.v_pool, torch.zeros((extra,) + tuple(b.v_pool.shape[1:]), dtype=b.v_pool.dtype)])
    bt2 = b.block_tables.copy()
    for s in range(sh.S):
        new = np.arange(b.num_blocks + s * nbp, b.num_blocks + (s + 1) * nbp)
        k[new] = b.k_pool[b.prefix_blocks]
        v[new] = b.v_pool[b.prefix_blocks]
        bt2[s, :nbp] = new
    d = to_dev(b)
    shared = gpu_attention(b, dev_tensors=d)
    d2 = dict(d, k=k.cuda(), v=v.cuda())
    copied = gpu_attention(b, dev_tensors=d2, bt=bt2)
    assert torch.equal(shared.view(torch.int16), copied.view(torch.int16))
    assert max_err(shared, oracle_attention(b)) <= TOL[shared.dtype]


def test_physical_relabelling_bit_identical():
    sh = synth.shrink(synth.CONFIGS["llama3_gqa_bs16"], S=4, len_fixed=None, len_uniform=(100, 900))
    b = synth.make_batch(sh)
    perm = np.random.default_rng(2).permutation(b.num_blocks)
    inv = torch.from_numpy(np.argsort(perm))
    d = to_dev(b)
    a = gpu_attention(b, dev_tensors=d)
    bt2 = np.where(b.block_tables >= 0, perm[np.maximum(b.block_tables, 0)], -1).astype(np.int32)
    d2 = dict(d, k=b.k_pool[inv].cuda(), v=b.v_pool[inv].cuda())
    c = gpu_attention(b, dev_tensors=d2, bt=bt2)
    assert torch.equal(a.view(torch.int16), c.view(torch.int16))


def test_tensor_core_group_path_equals_repeated_heads():
    """GQA on tensor cores vs the CUDA-core path on kv heads repeated G times."""
    sh = synth.shrink(synth.CONFIGS["llama3_gqa_bs16"], S=4, len_fixed=None, len_uniform=(1, 600))
    b = synth.make_batch(sh)
    ref = oracle_attention(b)
    gq = gpu_attention(b)
    G = sh.Hq // sh.Hkv
    d = to_dev(b)
    d2 = dict(d, k=d["k"].repeat_interleave(G, dim=1).contiguous(), v=d["v"].repeat_interleave(G, dim=1).contiguous())
    mh = gpu_attention(b, dev_tensors=d2)
    assert max_err(gq, ref) <= TOL[gq.dtype] and max_err(mh, ref) <= TOL[mh.dtype]


# --------------------------------------------------------------- device checks
def test_bad_block_id_is_reported_not_faulted():
    b = synth.make_batch(synth.CONFIGS["tiny"])
    bt = b.block_tables.copy()
    bt[2, 0] = 10_000
    d = to_dev(b)
    out = torch.empty_like(d["q"])
    pkv().paged_attention_decode(out, d["q"], d["k"], d["v"], torch.from_numpy(bt).cuda(), d["cl"])
    assert pkv().device_error() & pkv().binding.DEVERR_BLOCK_ID
    assert pkv().device_error() == 0                         # cleared


def test_bad_context_len_is_reported():
    b = synth.make_batch(synth.CONFIGS["tiny"])
    d = to_dev(b)
    out = torch.empty_like(d["q"])
    cl = torch.tensor([35, 16, 10_000, -3], dtype=torch.int32, device="cuda")
    pkv().paged_attention_decode(out, d["q"], d["k"], d["v"], d["bt"], cl)
    assert pkv().device_error() & pkv().binding.DEVERR_CONTEXT


def test_bad_slot_and_pair_are_reported():
    b = synth.make_batch(synth.CONFIGS["tiny"])
    d = to_dev(b)
    k0 = d["k"].clone()
    sm = torch.tensor([5, 10_000_000, -1, 7], dtype=torch.int64, device="cuda")
    pkv().kv_append(b.k_new.cuda(), b.v_new.cuda(), d["k"], d["v"], sm)
    assert pkv().device_error() & pkv().binding.DEVERR_SLOT
    pkv().block_copy(d["k"], d["v"], torch.tensor([[1, 99]], dtype=torch.int32, device="cuda"))
    assert pkv().device_error() & pkv().binding.DEVERR_BLOCK_ID
    assert not torch.equal(k0, d["k"])                        # the valid slots were written


# ------------------------------------------------------------ one decode step
def test_tiny_decode_step_end_to_end():
    """Allocator -> kv_append of one new token per sequence -> attention over L+1
    (the pages' decode step), both sides from the same inputs."""
    import paged_kv_cache_405_b200 as m
    b = synth.make_batch(synth.CONFIGS["tiny"])
    bs = b.shape.bs
    prod = m.BlockAllocator(b.num_blocks, bs, b.free_order)
    orc = oracle.Allocator(b.num_blocks, bs, b.free_order)
    for a in (prod, orc):
        for s in range(b.shape.S):
            a.seq_add(s)
            assert a.seq_append_slots(s, int(b.lens[s]))[0] == 0
    assert prod.seq_block_table(0)[1] == [7, 3, 9]
    slots, cows = [], []
    for s in range(b.shape.S):
        r1 = prod.seq_append_slots(s, 1)
        r2 = orc.seq_append_slots(s, 1)
        assert r1 == r2
        slots += r1[1]
        cows += r1[2]
    assert cows == [] and slots[0] == 9 * 16 + 3           # token 35 of seq 0: block 9, offset 3
    maxb = max(len(orc.seq_block_table(s)[1]) for s in range(4))
    bt = np.full((4, maxb), -1, np.int32)
    for s in range(4):
        t = prod.seq_block_table(s)[1]
        bt[s, :len(t)] = t
    lens = b.lens + 1
    kc, vc = b.k_pool.clone(), b.v_pool.clone()
    oracle.kv_append(kc, vc, b.k_new, b.v_new, slots)
    ref = oracle.paged_attention(b.q, kc, vc, bt, lens)
    d = to_dev(b)
    m.kv_append(b.k_new.cuda(), b.v_new.cuda(), d["k"], d["v"], torch.tensor(slots, device="cuda"))
    out = torch.empty_like(d["q"])
    m.paged_attention_decode(out, d["q"], d["k"], d["v"], torch.from_numpy(bt).cuda(),
                             torch.from_numpy(lens.astype(np.int32)).cuda())
    assert m.device_error() == 0
    assert torch.equal(d["k"].cpu(), kc) and torch.equal(d["v"].cpu(), vc)
    assert max_err(out, ref) <= TOL[torch.float32]
