"""Edge cases across the attention paths: the largest block sizes (128, 256
tokens), empty batches, and the maximum group size of the tensor-core path."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import TOL, gpu_attention, max_err, oracle_attention, to_dev
from test_gpu_chunk import chunk_case, run_chunk
from test_gpu_fp8 import fp8_pools

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bs", [128, 256])
@pytest.mark.parametrize("Hq,Hkv,dtype", [(4, 4, "bf16"), (16, 2, "bf16"), (4, 4, "f32"), (8, 2, "f16")])
def test_large_block_sizes(bs, Hq, Hkv, dtype):
    sh = synth.shrink(synth.CONFIGS["llama7b"], S=5, Hq=Hq, Hkv=Hkv, bs=bs, dtype=dtype, len_uniform=(1, 900),
                      seed=bs + Hq)
    b = synth.make_batch(sh, fill_unused=float("nan"))
    ref = oracle_attention(b)
    for P in (0, 64):
        out = gpu_attention(b, partition_size=P)
        assert max_err(out, ref) <= TOL[out.dtype], P


@pytest.mark.parametrize("bs", [128, 256])
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 2)])
def test_large_block_sizes_fp8(bs, Hq, Hkv):
    import paged_kv_cache_405_b200 as pkv
    sh = synth.shrink(synth.CONFIGS["llama7b"], S=5, Hq=Hq, Hkv=Hkv, bs=bs, len_uniform=(1, 900), seed=bs + Hq + 1)
    b = synth.make_batch(sh)
    ks, vs = 1 / 32, 1 / 8
    kc, vc = fp8_pools(b, 3, ks, vs)
    ref = oracle.paged_attention_kv(b.q, kc, vc, ks, vs, b.block_tables, b.lens, threads=oracle.max_threads())
    out = torch.full_like(b.q, float("nan"), device="cuda")
    pkv.paged_attention_decode_fp8(out, b.q.cuda(), kc.cuda(), vc.cuda(), torch.from_numpy(b.block_tables).cuda(),
                                   torch.from_numpy(b.lens.astype(np.int32)).cuda(), ks, vs, partition_size=64)
    assert pkv.device_error() == 0
    assert max_err(out, ref) <= TOL[out.dtype]


@pytest.mark.parametrize("bs", [128, 256])
def test_large_block_sizes_chunk(bs):
    import paged_kv_cache_405_b200 as pkv
    b, q, qs, max_n = chunk_case(16, 2, 128, bs, "bf16", seed=bs)
    out = run_chunk(b, q, qs, max_n, 64)
    assert pkv.device_error() == 0
    ref = oracle.paged_attention_chunk(q, b.k_pool, b.v_pool, b.block_tables, b.lens, qs,
                                       threads=oracle.max_threads())
    assert max_err(out, ref) <= TOL[out.dtype]


def test_group_of_sixteen_heads():
    """G = 16: every MMA row is a real query head."""
    sh = synth.shrink(synth.CONFIGS["llama7b"], S=4, Hq=32, Hkv=2, len_uniform=(1, 1500), seed=21)
    b = synth.make_batch(sh, fill_unused=float("nan"))
    ref = oracle_attention(b)
    for P in (0, 256):
        out = gpu_attention(b, partition_size=P)
        assert max_err(out, ref) <= TOL[out.dtype], P


def test_empty_batch_is_a_no_op():
    import paged_kv_cache_405_b200 as pkv
    sh = synth.shrink(synth.CONFIGS["llama7b"], S=3, Hq=8, Hkv=2, len_uniform=(1, 100), seed=4)
    b = synth.make_batch(sh)
    d = to_dev(b)
    before = pkv.launch_count()
    q0 = d["q"][:0]
    out0 = torch.empty_like(q0)
    pkv.paged_attention_decode(out0, q0, d["k"], d["v"], d["bt"][:0], d["cl"][:0])
    pkv.paged_attention_chunk(out0, q0, d["k"], d["v"], d["bt"][:0], d["cl"][:0],
                              torch.zeros(1, dtype=torch.int32, device="cuda"), 1)
    kc = torch.zeros(d["k"].shape, dtype=torch.uint8, device="cuda")
    pkv.paged_attention_decode_fp8(out0, q0, kc, kc, d["bt"][:0], d["cl"][:0], 1.0, 1.0)
    empty_new = torch.empty((0, sh.Hkv, sh.D), dtype=d["q"].dtype, device="cuda")
    pkv.kv_append(empty_new, empty_new, d["k"], d["v"], torch.empty(0, dtype=torch.int64, device="cuda"))
    pkv.block_copy(d["k"], d["v"], torch.empty((0, 2), dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert pkv.device_error() == 0
    assert pkv.launch_count() == before      # nothing to do, nothing launched
