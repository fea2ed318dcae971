"""Full-size parity: one step of every benchmark workload at its full size, in
the launch configuration the benchmark times (the benchmark's own workload
object: DecodeSession, the workload's partition size, shared-prefix groups,
copy-on-write forks, chunks, FP8 pools).

Every output row (every sequence or chunk row, every query head) is compared
with the oracle, which computes them all on the host cores; and both whole K/V
pools after the step are compared byte for byte with the oracle's
``block_copy`` and ``kv_append`` applied to the pools as they were before it
(the copy-on-write destinations of the beam workload, every appended row, and
no write anywhere else)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import TOL, max_err

pytestmark = pytest.mark.gpu

WORKLOADS = ["tiny", "llama7b", "llama13b_prefix", "llama3_gqa_bs16", "llama3_gqa_bs32", "longctx_beam", "spec_verify",
             "llama7b_fp8", "llama3_gqa_fp8"]


def _bits(t: torch.Tensor) -> torch.Tensor:
    return t.view({1: torch.uint8, 2: torch.int16, 4: torch.int32}[t.element_size()])


@pytest.mark.parametrize("cfg", WORKLOADS)
def test_full_size_step_every_output_and_whole_pools(cfg):
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
    torch.cuda.synchronize()
    k0, v0 = wl.session.k_pool.cpu(), wl.session.v_pool.cpu()      # the pools before the step
    out = torch.full((Tq, shape.Hq, shape.D), float("nan"), dtype=dt, device=dev)
    wl.launch(d, q.to(dev), kn.to(dev), vn.to(dev), out)
    torch.cuda.synchronize()
    assert m.device_error() == 0
    kc, vc = wl.session.k_pool.cpu(), wl.session.v_pool.cpu()
    got = out.cpu()
    del out, d, wl
    torch.cuda.empty_cache()

    # the pools: the oracle's copies, then its appends, on the pre-step pools
    if shape.beams:
        assert len(p.cow_pairs) == shape.S * (shape.beams - 1)     # 3 copies per parent (4 beams)
    oracle.block_copy(k0, v0, p.cow_pairs)
    if shape.kv_fp8:
        oracle.kv_append_fp8(k0.numpy(), v0.numpy(), kn, vn, shape.kv_scale, shape.kv_scale, p.slot_mapping)
    else:
        oracle.kv_append(k0, v0, kn, vn, p.slot_mapping)
    assert torch.equal(_bits(kc), _bits(k0)), "K pool differs from the oracle's copies + appends"
    assert torch.equal(_bits(vc), _bits(v0)), "V pool differs from the oracle's copies + appends"
    del k0, v0

    # every output row
    lens = np.asarray(p.lens)
    th = oracle.max_threads()
    if shape.chunk:
        ref = oracle.paged_attention_chunk(q, kc, vc, p.block_tables, lens, p.query_start, threads=th)
    elif shape.kv_fp8:
        ref = oracle.paged_attention_kv(q, kc.numpy(), vc.numpy(), shape.kv_scale, shape.kv_scale, p.block_tables,
                                        lens, threads=th)
    else:
        ref = oracle.paged_attention(q, kc, vc, p.block_tables, lens, threads=th)
    assert ref.shape == tuple(got.shape)
    assert max_err(got, ref) <= TOL[dt]
