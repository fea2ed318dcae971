"""The decode entry point that allocates nothing, checked against the regular one.

pkv_paged_attention_decode_static serves callers that cannot allocate device
memory (an allocator that owns all of it, a plug-in restricted to the buffers
it is handed, a step loop that must not hit a synchronising cudaMalloc): its
split-K scratch is a fixed buffer compiled into the library.  Here it is
called through the C ABI twice in a row, on inputs that use split-K, and each
result is compared with pkv_paged_attention_decode given a normal workspace,
within the attention tolerance of the other GPU tests.  This file runs last so
that a failure here leaves every other test already run.
"""
import numpy as np
import pytest
import torch

import synth
from gpu_helpers import TOL, max_err, oracle_attention, to_dev

pytestmark = pytest.mark.gpu


def both(batch, partition_size):
    import paged_kv_cache_405_b200 as pkv
    d = to_dev(batch)
    ref = torch.full_like(d["q"], float("nan"))
    pkv.paged_attention_decode(ref, d["q"], d["k"], d["v"], d["bt"], d["cl"], partition_size=partition_size)
    got = torch.full_like(d["q"], float("nan"))
    pkv.paged_attention_decode_static(got, d["q"], d["k"], d["v"], d["bt"], d["cl"], partition_size=partition_size)
    assert pkv.device_error() == 0
    return ref, got


def test_static_scratch_matches_workspace_call_twice_in_a_row():
    # first call: grouped-query heads on tensor cores, 100+ partitions of 64 tokens
    a = synth.make_batch(synth.shrink(synth.CONFIGS["longctx_beam"], S=3, Hq=16, Hkv=2, len_fixed=None,
                                      len_uniform=(3000, 7000)), fill_unused=float("nan"))
    # second call: multi-head attention on CUDA cores, different shapes, so stale
    # partials from the first call sit in the shared buffer
    b = synth.make_batch(synth.shrink(synth.CONFIGS["llama7b"], S=9, Hq=8, Hkv=8, len_uniform=(1, 1500)),
                         fill_unused=float("nan"))
    for batch, P in ((a, 64), (b, 128)):
        ref, got = both(batch, P)
        assert max_err(got, oracle_attention(batch)) <= TOL[got.dtype]
        assert (got.float() - ref.float()).abs().max().item() <= TOL[got.dtype]


def test_static_scratch_rejects_oversized_calls():
    import paged_kv_cache_405_b200 as pkv
    b = synth.make_batch(synth.shrink(synth.CONFIGS["llama7b"], S=4, Hq=8, Hkv=8, len_uniform=(1, 64)))
    d = to_dev(b)
    out = torch.zeros_like(d["q"])
    # 4 seqs x 8 heads x 8192 partitions of 16 tokens x 130 floats = 136 MB: a
    # valid call otherwise, but beyond the 64 MiB buffer
    bt = torch.zeros((4, 8192), dtype=torch.int32, device="cuda")
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.paged_attention_decode_static(out, d["q"], d["k"], d["v"], bt, d["cl"], partition_size=16)
    assert "scratch" in str(e.value)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0            # nothing was launched
