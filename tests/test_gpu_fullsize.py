"""Full-size parity: one step of every benchmark workload at its full size, in
the launch configuration the benchmark times (the benchmark's own workload
object: DecodeSession, the workload's partition size, shared-prefix groups,
copy-on-write forks, chunks, FP8 pools), checked on sampled outputs the
oracle computes one by one, and on sampled appended rows byte for byte."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import TOL, max_err

pytestmark = pytest.mark.gpu

WORKLOADS = ["llama7b", "llama13b_prefix", "llama3_gqa_bs16", "llama3_gqa_bs32", "longctx_beam", "spec_verify",
             "llama7b_fp8", "llama3_gqa_fp8"]


@pytest.mark.parametrize("cfg", WORKLOADS)
def test_full_size_step_on_sampled_outputs(cfg):
    import bench
    import paged_kv_cache_405_b200 as m
    shape = synth.CONFIGS[cfg]
    dev = torch.device("cuda")
    wl = bench.Workload(shape, shape.seed, dev, 0)
    p = wl.plan()
    d = wl.to_device(p)
    dt = synth.DTYPES[shape.dtype]
    T = len(p.slot_mapping)                        # tokens written this step
    Tq = T if shape.chunk else len(p.seq_ids)      # query rows
    g = torch.Generator().manual_seed(4242)
    q = synth.randn((Tq, shape.Hq, shape.D), g, dt, "cpu")
    kn = synth.randn((T, shape.Hkv, shape.D), g, dt, "cpu")
    vn = synth.randn((T, shape.Hkv, shape.D), g, dt, "cpu")
    out = torch.full((Tq, shape.Hq, shape.D), float("nan"), dtype=dt, device=dev)
    wl.launch(d, q.to(dev), kn.to(dev), vn.to(dev), out)
    torch.cuda.synchronize()
    assert m.device_error() == 0
    kc, vc = wl.session.k_pool.cpu(), wl.session.v_pool.cpu()

    rng = np.random.default_rng(99)
    bs = shape.bs
    # appended rows, byte for byte (the quantized codes for FP8 pools)
    for i in rng.choice(T, size=min(T, 24), replace=False).tolist():
        sl = int(p.slot_mapping[i])
        blk, off = sl // bs, sl % bs
        if shape.kv_fp8:
            assert np.array_equal(kc[blk, :, off].numpy(), oracle.quantize_e4m3(kn[i], shape.kv_scale))
            assert np.array_equal(vc[blk, :, off].numpy(), oracle.quantize_e4m3(vn[i], shape.kv_scale))
        else:
            assert torch.equal(kc[blk, :, off].view(torch.int16), kn[i].view(torch.int16))
            assert torch.equal(vc[blk, :, off].view(torch.int16), vn[i].view(torch.int16))

    # sampled outputs: the longest context, the first and last rows, and random ones
    lens = np.asarray(p.lens)
    if shape.chunk:
        qs = np.asarray(p.query_start)
        seqs = [int(np.argmax(lens)), 0, len(lens) - 1] + rng.choice(len(lens), size=9).tolist()
        rows = [int(qs[s] + rng.integers(0, qs[s + 1] - qs[s])) for s in seqs] + [int(qs[-1]) - 1]
    else:
        rows = [int(np.argmax(lens)), 0, Tq - 1] + rng.choice(Tq, size=9).tolist()
    items = [(r, int(rng.integers(0, shape.Hq))) for r in rows]
    th = oracle.max_threads()
    if shape.chunk:
        ref = oracle.paged_attention_chunk(q, kc, vc, p.block_tables, lens, p.query_start, items=items, threads=th)
    elif shape.kv_fp8:
        ref = oracle.paged_attention_kv(q, kc.numpy(), vc.numpy(), shape.kv_scale, shape.kv_scale, p.block_tables,
                                        lens, items=items, threads=th)
    else:
        ref = oracle.paged_attention(q, kc, vc, p.block_tables, lens, items=items, threads=th)
    got = torch.stack([out[r, h] for r, h in items]).cpu()
    assert max_err(got, ref) <= TOL[dt]
