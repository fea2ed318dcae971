"""Split-K partials and their merge, checked against the oracle with a
workspace full of garbage (its contents need no initialisation), across
repeated calls on the same workspace (bit-identical results), for partition
counts from 2 to 75 and for the 16-bit and FP8 kernels."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import TOL, max_err, oracle_attention, to_dev
from test_gpu_fp8 import fp8_pools

pytestmark = pytest.mark.gpu


def garbage_workspace(q, bt, bs, P, seed):
    import paged_kv_cache_405_b200 as pkv
    n = pkv.attention_workspace_bytes(q.shape[0], q.shape[1], q.shape[2], bt.shape[1] * bs, P)
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randint(0, 256, (max(n, 256),), dtype=torch.uint8, device="cuda", generator=g)


@pytest.mark.parametrize("Hq,Hkv,dtype", [(8, 8, "bf16"), (16, 2, "bf16"), (8, 8, "f32"), (8, 1, "f16")])
@pytest.mark.parametrize("P", [16, 32, 64, 512])
def test_merge_with_garbage_workspace_and_repeated_calls(Hq, Hkv, dtype, P):
    import paged_kv_cache_405_b200 as pkv
    sh = synth.shrink(synth.CONFIGS["llama7b"], S=9, Hq=Hq, Hkv=Hkv, dtype=dtype, len_uniform=(0, 1000),
                      seed=P + Hq)
    b = synth.make_batch(sh, fill_unused=float("nan"))
    ref = oracle_attention(b)
    d = to_dev(b)
    ws = garbage_workspace(d["q"], d["bt"], sh.bs, P, P)
    outs = []
    for _ in range(3):                      # the same workspace, one call after another
        out = torch.full_like(d["q"], float("nan"))
        pkv.paged_attention_decode(out, d["q"], d["k"], d["v"], d["bt"], d["cl"], partition_size=P, workspace=ws)
        assert pkv.device_error() == 0
        assert max_err(out, ref) <= TOL[out.dtype]
        outs.append(out)
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])   # deterministic


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 2)])
def test_merge_fp8(Hq, Hkv):
    import paged_kv_cache_405_b200 as pkv
    sh = synth.shrink(synth.CONFIGS["llama7b"], S=7, Hq=Hq, Hkv=Hkv, len_uniform=(1, 1200), seed=Hq)
    b = synth.make_batch(sh)
    ks, vs = 1 / 32, 1 / 8
    kc, vc = fp8_pools(b, 6, ks, vs)
    ref = oracle.paged_attention_kv(b.q, kc, vc, ks, vs, b.block_tables, b.lens, threads=oracle.max_threads())
    q, bt = b.q.cuda(), torch.from_numpy(b.block_tables).cuda()
    cl = torch.from_numpy(b.lens.astype(np.int32)).cuda()
    for P in (64, 16):                      # 20 and 80 partition slots
        ws = garbage_workspace(q, bt, sh.bs, P, 3)
        out = torch.full_like(q, float("nan"))
        pkv.paged_attention_decode_fp8(out, q, kc.cuda(), vc.cuda(), bt, cl, ks, vs, partition_size=P, workspace=ws)
        assert pkv.device_error() == 0
        assert max_err(out, ref) <= TOL[out.dtype], P
