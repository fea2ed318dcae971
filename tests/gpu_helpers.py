"""Helpers for the GPU parity tests: run the CUDA path and the oracle on the
same seeded inputs and compare."""
import numpy as np
import torch

import oracle
import synth

# Attention tolerance, max |gpu - oracle| over all outputs: fp32 outputs 5e-3,
# 16-bit outputs 2e-2 (fp32 accumulation on the GPU, one rounding at the end).
TOL = {torch.float32: 5e-3, torch.bfloat16: 2e-2, torch.float16: 2e-2}


def to_dev(batch: synth.Batch, dev="cuda"):
    return dict(
        q=batch.q.to(dev), k=batch.k_pool.to(dev), v=batch.v_pool.to(dev),
        bt=torch.from_numpy(batch.block_tables).to(dev),
        cl=torch.from_numpy(batch.lens.astype(np.int32)).to(dev),
    )


def gpu_attention(batch, lens=None, partition_size=0, dev_tensors=None, bt=None):
    import paged_kv_cache_405_b200 as pkv
    d = dev_tensors or to_dev(batch)
    cl = d["cl"] if lens is None else torch.as_tensor(np.asarray(lens, dtype=np.int32)).cuda()
    btt = d["bt"] if bt is None else torch.as_tensor(np.ascontiguousarray(bt, dtype=np.int32)).cuda()
    out = torch.full_like(d["q"], float("nan"))
    pkv.paged_attention_decode(out, d["q"], d["k"], d["v"], btt, cl, partition_size=partition_size)
    assert pkv.device_error() == 0
    return out


def oracle_attention(batch, lens=None, bt=None, items=None, k=None, v=None, q=None):
    return oracle.paged_attention(batch.q if q is None else q,
                                  batch.k_pool if k is None else k,
                                  batch.v_pool if v is None else v,
                                  batch.block_tables if bt is None else bt,
                                  batch.lens if lens is None else lens, items=items,
                                  threads=oracle.max_threads())


def max_err(gpu_out: torch.Tensor, ref: np.ndarray) -> float:
    g = gpu_out.double().cpu().numpy()
    assert g.shape == ref.shape
    assert np.isfinite(g).all(), "non-finite output"
    return float(np.abs(g - ref).max())
