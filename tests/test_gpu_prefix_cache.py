"""Automatic prefix caching through DecodeSession on the device: a prompt
whose leading full blocks are cached reuses their K/V as written by the
earlier prompt (only its other tokens are appended), a freed sequence's
cached blocks are revived by the same prompt, and decode attention over the
reused blocks matches the oracle on each sequence's own prompt."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import TOL, max_err

pytestmark = pytest.mark.gpu

Hq, Hkv, D, BS, NB, MAXB = 8, 2, 128, 16, 48, 8


def prompt_kv(tokens):
    """K/V of each prompt position as a function of the whole prefix up to it
    (what a model's K/V depend on), so equal prefixes give equal rows."""
    ks, vs = [], []
    h = 1469598103934665603
    for t in tokens:
        h = ((h ^ int(t)) * 1099511628211) % (1 << 61)
        g = torch.Generator().manual_seed(h)
        ks.append(torch.randn(Hkv, D, generator=g))
        vs.append(torch.randn(Hkv, D, generator=g))
    return torch.stack(ks).to(torch.bfloat16), torch.stack(vs).to(torch.bfloat16)


def write(ss, mirror, kv, slots):
    import paged_kv_cache_405_b200 as m
    k, v = kv
    if len(slots):
        sl = torch.from_numpy(np.asarray(slots, dtype=np.int64))
        m.kv_append(k.cuda(), v.cuda(), ss.k_pool, ss.v_pool, sl.cuda())
        oracle.kv_append(mirror[0], mirror[1], k, v, sl)


def step(ss, mirror, seqs, seed):
    import paged_kv_cache_405_b200 as m
    g = torch.Generator().manual_seed(seed)
    n = len(seqs)
    q = torch.randn(n, Hq, D, generator=g).to(torch.bfloat16)
    kn = torch.randn(n, Hkv, D, generator=g).to(torch.bfloat16)
    vn = torch.randn(n, Hkv, D, generator=g).to(torch.bfloat16)
    p = ss.plan(seqs)
    out = torch.empty(n, Hq, D, dtype=torch.bfloat16, device="cuda")
    ss.launch(ss.to_device(p), q.cuda(), kn.cuda(), vn.cuda(), out)
    oracle.block_copy(mirror[0], mirror[1], p.cow_pairs)
    oracle.kv_append(mirror[0], mirror[1], kn, vn, p.slot_mapping)
    ref = oracle.paged_attention(q, mirror[0], mirror[1], p.block_tables, p.lens)
    assert m.device_error() == 0
    assert max_err(out, ref) <= TOL[out.dtype]


def test_cached_prompt_blocks_serve_attention():
    import paged_kv_cache_405_b200 as m
    rng = np.random.default_rng(5)
    base = rng.integers(0, 32000, 40).tolist()
    A = base + rng.integers(0, 32000, 10).tolist()            # 50 tokens: 3 full blocks + 2
    B = base[:32] + rng.integers(0, 32000, 20).tolist()       # shares A's first two blocks
    k = torch.zeros(NB, Hkv, BS, D, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    mirror = (k.cpu(), v.cpu())
    ss = m.DecodeSession(k, v, Hq, MAXB, max_batch=4, prefix_caching=True, share_prefixes=False)

    n_a, slots_a = ss.add_prompt(0, A)
    assert n_a == 0 and len(slots_a) == len(A)
    write(ss, mirror, prompt_kv(A), slots_a)
    n_b, slots_b = ss.add_prompt(1, B)
    assert n_b == 32 and len(slots_b) == len(B) - 32          # two cached blocks reused
    kb, vb = prompt_kv(B)
    write(ss, mirror, (kb[32:], vb[32:]), slots_b)
    assert ss.table(1)[0][:2] == ss.table(0)[0][:2]
    st = ss.cache_stats()
    assert st["hits"] == 2

    step(ss, mirror, [0, 1], seed=1)                          # both write their own partial last block
    # The reused rows hold exactly what B's own prompt would have written.
    bt_b = ss.table(1)[0]
    for t in range(32):
        blk, off = bt_b[t // BS], t % BS
        assert torch.equal(k[blk, :, off].cpu(), kb[t]) and torch.equal(v[blk, :, off].cpu(), vb[t])

    ss.free(0)                                                # A's third block stays cached, evictable
    n_c, slots_c = ss.add_prompt(2, A)
    assert n_c == 48 and len(slots_c) == len(A) - 48          # revived: all three full blocks
    ka, va = prompt_kv(A)
    write(ss, mirror, (ka[48:], va[48:]), slots_c)
    step(ss, mirror, [1, 2], seed=2)
    assert ss.cache_stats()["hits"] == 5
    assert torch.equal(k.cpu(), mirror[0]) and torch.equal(v.cpu(), mirror[1])
