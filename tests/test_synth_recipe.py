"""The synthetic workloads follow the stated input recipe: length
distributions per workload, the worked example's blocks for the tiny
workload, N(0,1) values, blocks handed out in sequence order from one seeded
permutation (prompt first), and the long-context workload's partial last
block."""
import math

import numpy as np
import torch

import synth


def lengths(name):
    sh = synth.CONFIGS[name]
    return synth._lengths(sh, np.random.default_rng(sh.seed))


def test_length_recipes():
    assert lengths("tiny").tolist() == [35, 16, 1, 50]
    for name in ("llama7b", "llama7b_fp8"):
        L = lengths(name)
        assert len(L) == 64 and L.min() >= 128 and L.max() <= 2048
    L = lengths("spec_verify")
    assert len(L) == 64 and L.min() >= 1024 and L.max() <= 8192
    for name in ("llama3_gqa_bs16", "llama3_gqa_bs32", "llama3_gqa_fp8"):
        assert lengths(name).tolist() == [8192] * 128
    L = lengths("longctx_beam")
    assert L.tolist() == [100_000] * 8
    assert 100_000 - (100_000 // 64) * 64 == 32          # the last of 1563 blocks holds 32 tokens


def test_shared_prompt_plus_log_normal_suffix():
    """512-token prompt + suffix with ln L ~ N(ln 300, 1), rounded, clipped to [1, 4096]."""
    L = lengths("llama13b_prefix")
    suf = L - 512
    assert len(L) == 256 and suf.min() >= 1 and suf.max() <= 4096
    # median of 256 draws of a log-normal with median 300: within a loose band
    assert 200 <= np.median(suf) <= 450
    # log of the suffix has spread near 1 (the stated sigma)
    assert 0.8 <= np.std(np.log(suf)) <= 1.2


def test_tiny_batch_blocks_and_values():
    b = synth.make_batch(synth.CONFIGS["tiny"])
    assert b.free_order[:3].tolist() == [7, 3, 9]
    assert sorted(b.free_order.tolist()) == list(range(32))
    assert b.block_tables[0, :3].tolist() == [7, 3, 9]
    # sequences take the next blocks of the same order, in sequence order
    used = [int(x) for s in range(4) for x in b.block_tables[s] if x >= 0]
    assert used == b.free_order[:len(used)].tolist()
    v = b.k_pool.double()
    assert abs(float(v.mean())) < 0.05 and abs(float(v.std()) - 1.0) < 0.05     # N(0,1) values


def test_prompt_blocks_come_first_and_are_shared():
    sh = synth.shrink(synth.CONFIGS["llama13b_prefix"], S=5, Hq=1, Hkv=1, D=64)
    b = synth.make_batch(sh)
    nb_prefix = 512 // 16
    prompt = b.free_order[:nb_prefix].tolist()
    for s in range(sh.S):
        assert b.block_tables[s, :nb_prefix].tolist() == prompt
    own = [int(x) for s in range(sh.S) for x in b.block_tables[s, nb_prefix:] if x >= 0]
    assert own == b.free_order[nb_prefix:nb_prefix + len(own)].tolist()
    assert math.isclose(float(b.k_pool.float().std()), 1.0, rel_tol=0.05)
    assert b.k_pool.dtype == torch.bfloat16
