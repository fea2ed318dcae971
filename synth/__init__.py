"""Seeded synthetic inputs for paged decode attention.

This module is the only code shared by the oracle side (``oracle/``, the tests)
and the CUDA side (the package, ``bench.py``).  It draws random numbers and lays
out input structure -- sequence lengths, which physical blocks each sequence is
handed, the values in the K/V pools -- and holds none of the method's
arithmetic: no slot translation, no attention, no allocator logic.

Workload shapes follow the pages' workloads (Llama-7B/13B-shaped heads,
block_size 16, a shared system prompt, beam-style sharing, 100k-token
contexts); see ``CONFIGS``.  Every tensor is produced from a
``torch.Generator`` seeded per config, on the device asked for, so a given
(config, seed, device) always yields the same bytes.

Pool layout (the input format both sides read): ``[num_blocks, num_kv_heads,
block_size, head_dim]``, row-major.  Block tables are ``int32 [S, max_blocks]``
padded with -1.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


@dataclass
class Shape:
    """Static description of one decode workload."""

    name: str
    S: int                      # sequences in the batch
    Hq: int                     # query heads
    Hkv: int                    # kv heads (Hq % Hkv == 0)
    D: int                      # head dim
    bs: int                     # tokens per block
    dtype: str                  # "f32" | "bf16" | "f16"
    seed: int
    lens: Optional[list] = None         # explicit lengths before the step
    len_uniform: Optional[tuple] = None  # (lo, hi) inclusive
    len_fixed: Optional[int] = None
    prefix: int = 0                     # shared prefix tokens (stored once)
    suffix_lognormal: Optional[tuple] = None  # (median, sigma, lo, hi)
    num_blocks: Optional[int] = None    # explicit pool size
    pool_factor: float = 1.2            # pool = factor x need (plus reserve)
    reserve_tokens: int = 64            # growth room per sequence
    partition_size: int = 0             # 0 = library's choice
    beams: int = 0                      # beams forked per sequence
    pinned_seq0: Optional[list] = None  # explicit physical blocks of seq 0
    chunk: int = 0                      # new tokens per sequence per step (causal chunk); 0 = decode
    kv_fp8: bool = False                # pools of FP8 E4M3 codes (values = code x kv_scale)
    kv_scale: float = 1.0 / 32          # k_scale = v_scale for FP8 pools
    description: str = ""


CONFIGS = {
    # 4 seqs, lengths {35,16,1,50}, 4 q = 4 kv heads, head_dim 64, bs 16,
    # 32-block pool; seq 0 owns physical blocks 7, 3, 9 (the pages' worked
    # example); fp32 values.
    "tiny": Shape("tiny", S=4, Hq=4, Hkv=4, D=64, bs=16, dtype="f32", seed=0,
                  lens=[35, 16, 1, 50], num_blocks=32, pinned_seq0=[7, 3, 9],
                  description="tiny paged decode: 4 seqs, lens {35,16,1,50}, 4 heads x 64, bs 16, 32 blocks, fp32"),
    # Llama-2-7B-shaped layer: batch 64, 32 heads x 128, lengths U[128, 2048].
    "llama7b": Shape("llama7b", S=64, Hq=32, Hkv=32, D=128, bs=16, dtype="bf16", seed=1,
                     len_uniform=(128, 2048),
                     description="Llama-2-7B-shaped decode: batch 64, MHA 32x128, bf16, bs 16, ctx U[128,2048]"),
    # LLaMA-13B-shaped layer: batch 256, 40 heads x 128, one 512-token system
    # prompt shared by every sequence, private log-normal suffix.
    "llama13b_prefix": Shape("llama13b_prefix", S=256, Hq=40, Hkv=40, D=128, bs=16, dtype="bf16",
                             seed=3, prefix=512, suffix_lognormal=(300.0, 1.0, 1, 4096),
                             description="LLaMA-13B-shaped decode, 512-token shared prefix: batch 256, MHA 40x128, bf16, bs 16"),
    # Llama-3-8B-shaped GQA layer: batch 128, 32 q / 8 kv heads, 8192 tokens.
    "llama3_gqa_bs16": Shape("llama3_gqa_bs16", S=128, Hq=32, Hkv=8, D=128, bs=16, dtype="bf16",
                             seed=5, len_fixed=8192, pool_factor=1.0,
                             description="Llama-3-8B-shaped GQA decode: batch 128, 32q/8kv x 128, bf16, ctx 8192, bs 16"),
    "llama3_gqa_bs32": Shape("llama3_gqa_bs32", S=128, Hq=32, Hkv=8, D=128, bs=32, dtype="bf16",
                             seed=5, len_fixed=8192, pool_factor=1.0,
                             description="Llama-3-8B-shaped GQA decode: batch 128, 32q/8kv x 128, bf16, ctx 8192, bs 32"),
    # Speculative verification (an extension beyond the five decode
    # workloads): Llama-3-8B-shaped GQA, batch 64, 4 draft tokens per
    # sequence attending causally to contexts of U[1024, 8192].
    "spec_verify": Shape("spec_verify", S=64, Hq=32, Hkv=8, D=128, bs=16, dtype="bf16", seed=7,
                         len_uniform=(1024, 8192), chunk=4,
                         description="speculative verification: batch 64 x 4 draft tokens, 32q/8kv x 128, bf16, bs 16, ctx U[1024,8192]"),
    # FP8 E4M3 pools (extensions): the Llama-2-7B and Llama-3-8B decode
    # workloads with K/V stored as 1-byte codes.
    "llama7b_fp8": Shape("llama7b_fp8", S=64, Hq=32, Hkv=32, D=128, bs=16, dtype="bf16", seed=1,
                         len_uniform=(128, 2048), kv_fp8=True,
                         description="Llama-2-7B-shaped decode over FP8 E4M3 pools: batch 64, MHA 32x128, bf16 q/out, bs 16"),
    "llama3_gqa_fp8": Shape("llama3_gqa_fp8", S=128, Hq=32, Hkv=8, D=128, bs=16, dtype="bf16", seed=5,
                            len_fixed=8192, pool_factor=1.0, kv_fp8=True,
                            description="Llama-3-8B-shaped GQA decode over FP8 E4M3 pools: batch 128, 32q/8kv x 128, ctx 8192"),
    # Long context + beams: 8 x 100k tokens, 64 q / 8 kv heads, bs 64,
    # split over 512-token partitions; 4 beams fork each sequence.
    "longctx_beam": Shape("longctx_beam", S=8, Hq=64, Hkv=8, D=128, bs=64, dtype="bf16", seed=6,
                          len_fixed=100_000, pool_factor=1.0, partition_size=512, beams=4,
                          description="long context + beam COW: 8 x 100k tokens, 64q/8kv x 128, bf16, bs 64, split-K 512, 4 beams"),
}


def shrink(shape: Shape, **over) -> Shape:
    """A copy of ``shape`` with fields replaced (for small parity cases)."""
    d = dict(shape.__dict__)
    d.update(over)
    return Shape(**d)


@dataclass
class Batch:
    """One decode batch: pools, block tables, lengths, step inputs."""

    shape: Shape
    num_blocks: int
    lens: np.ndarray                 # int64 [S], tokens cached before the step
    block_tables: np.ndarray         # int32 [S, maxB], -1 padded
    free_order: np.ndarray           # int32 [NB]; blocks handed out front-first
    prefix_blocks: np.ndarray        # int32 [n] shared prefix blocks (may be empty)
    k_pool: torch.Tensor             # [NB, Hkv, bs, D]
    v_pool: torch.Tensor
    q: torch.Tensor                  # [S, Hq, D]
    k_new: torch.Tensor              # [S, Hkv, D]  (one new token per sequence)
    v_new: torch.Tensor
    extra: dict = field(default_factory=dict)

    @property
    def max_blocks(self) -> int:
        return int(self.block_tables.shape[1])


def _lengths(shape: Shape, rng: np.random.Generator) -> np.ndarray:
    if shape.lens is not None:
        return np.asarray(shape.lens, dtype=np.int64)
    if shape.len_fixed is not None:
        return np.full(shape.S, shape.len_fixed, dtype=np.int64)
    if shape.len_uniform is not None:
        lo, hi = shape.len_uniform
        return rng.integers(lo, hi + 1, size=shape.S).astype(np.int64)
    if shape.suffix_lognormal is not None:
        med, sigma, lo, hi = shape.suffix_lognormal
        suf = np.rint(np.exp(rng.normal(math.log(med), sigma, size=shape.S)))
        suf = np.clip(suf, lo, hi).astype(np.int64)
        return suf + shape.prefix
    raise ValueError("shape has no length recipe")


def randn(shape, gen: torch.Generator, dtype: torch.dtype, device, chunk: int = 1 << 27) -> torch.Tensor:
    """N(0,1) samples drawn in fp32 and rounded once (RNE) to ``dtype``."""
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=dtype, device=device)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        out[s:e] = torch.randn(e - s, generator=gen, dtype=torch.float32, device=device).to(dtype)
    return out.view(*shape)


def fp8_codes(shape, gen: torch.Generator, scale: float, device, chunk: int = 1 << 27) -> torch.Tensor:
    """uint8 E4M3 codes of N(0,1) samples divided by ``scale`` (torch cast)."""
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=torch.uint8, device=device)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        x = torch.randn(e - s, generator=gen, dtype=torch.float32, device=device) / scale
        out[s:e] = x.to(torch.float8_e4m3fn).view(torch.uint8)
    return out.view(*shape)


def make_batch(shape: Shape, device="cpu", seed: Optional[int] = None,
               value_scale: float = 1.0, fill_unused=None) -> Batch:
    """Build the batch for ``shape``.

    Block hand-out: a seeded permutation of the pool is the free order; the
    prefix (if any) takes the first ``ceil(prefix/bs)`` entries, then each
    sequence in turn takes the next ``ceil(own tokens/bs)`` entries.  For the
    tiny config seq 0's blocks are pinned to the given list and the rest of
    the pool is permuted with ``numpy.random.default_rng(seed)``.

    ``fill_unused`` (a float, e.g. NaN) overwrites every pool row that no
    sequence covers, to check that a kernel never reads past a context.
    """
    seed = shape.seed if seed is None else seed
    rng = np.random.default_rng(seed)
    lens = _lengths(shape, rng)
    bs = shape.bs
    nb_prefix = -(-shape.prefix // bs) if shape.prefix else 0
    own = lens - shape.prefix
    nb_own = -(-own // bs)
    need = nb_prefix + int(nb_own.sum())
    if shape.num_blocks is not None:
        NB = shape.num_blocks
    else:
        reserve = shape.S * (-(-shape.reserve_tokens // bs) + 1)
        if shape.beams:
            reserve += shape.S * shape.beams * (-(-shape.reserve_tokens // bs) + 1)
        NB = int(math.ceil(shape.pool_factor * need)) + reserve
    if shape.pinned_seq0 is not None:
        pinned = list(shape.pinned_seq0)
        rest = np.array([b for b in range(NB) if b not in pinned], dtype=np.int64)
        free_order = np.concatenate([np.array(pinned, dtype=np.int64), rng.permutation(rest)])
    else:
        free_order = rng.permutation(NB)
    free_order = free_order.astype(np.int32)

    max_nb = nb_prefix + int(nb_own.max()) + (-(-shape.reserve_tokens // bs)) + 1
    bt = np.full((shape.S, max_nb), -1, dtype=np.int32)
    cur = 0
    prefix_blocks = free_order[:nb_prefix].copy()
    cur += nb_prefix
    for s in range(shape.S):
        bt[s, :nb_prefix] = prefix_blocks
        n = int(nb_own[s])
        bt[s, nb_prefix:nb_prefix + n] = free_order[cur:cur + n]
        cur += n

    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    dt = DTYPES[shape.dtype]
    pshape = (NB, shape.Hkv, bs, shape.D)
    if shape.kv_fp8:   # codes of N(0,1) values / kv_scale, cast by torch's float8_e4m3fn
        k_pool = fp8_codes(pshape, gen, shape.kv_scale, device)
        v_pool = fp8_codes(pshape, gen, shape.kv_scale, device)
    else:
        k_pool = randn(pshape, gen, dt, device)
        v_pool = randn(pshape, gen, dt, device)
    q = randn((shape.S, shape.Hq, shape.D), gen, dt, device)
    k_new = randn((shape.S, shape.Hkv, shape.D), gen, dt, device)
    v_new = randn((shape.S, shape.Hkv, shape.D), gen, dt, device)
    if value_scale != 1.0:
        for t in ((q, k_new, v_new) if shape.kv_fp8 else (k_pool, v_pool, q, k_new, v_new)):
            t.copy_((t.float() * value_scale).to(dt))
    if fill_unused is not None:
        covered = torch.zeros((NB, bs), dtype=torch.bool)
        for s in range(shape.S):
            L = int(lens[s])
            nb = -(-L // bs)
            for j in range(nb):
                blk = int(bt[s, j])
                covered[blk, : min(bs, L - j * bs)] = True
        mask = (~covered).to(device)
        k_pool.masked_fill_(mask[:, None, :, None], fill_unused)
        v_pool.masked_fill_(mask[:, None, :, None], fill_unused)
    return Batch(shape=shape, num_blocks=NB, lens=lens, block_tables=bt, free_order=free_order,
                 prefix_blocks=prefix_blocks, k_pool=k_pool, v_pool=v_pool, q=q,
                 k_new=k_new, v_new=v_new)


def step_inputs(shape: Shape, step: int, device="cpu", seed: Optional[int] = None):
    """Fresh (q, k_new, v_new) for decode step ``step`` of a batch."""
    seed = shape.seed if seed is None else seed
    gen = torch.Generator(device=device)
    gen.manual_seed(1_000_003 * (seed + 1) + step)
    dt = DTYPES[shape.dtype]
    q = randn((shape.S, shape.Hq, shape.D), gen, dt, device)
    k_new = randn((shape.S, shape.Hkv, shape.D), gen, dt, device)
    v_new = randn((shape.S, shape.Hkv, shape.D), gen, dt, device)
    return q, k_new, v_new


def random_ops(seed: int, n_ops: int, max_seqs: int = 4, max_append: int = 5):
    """A seeded random sequence of allocator operations (for model checking).

    Each op is a tuple: ("add", sid) | ("append", sid, n) | ("fork", parent, child)
    | ("share", sid, donor_sid, ntok) | ("free", sid).  Operations may be invalid
    (unknown ids, ...); both allocators must agree on the status.
    """
    rng = np.random.default_rng(seed)
    ops = []
    for _ in range(n_ops):
        kind = rng.choice(["add", "append", "append", "append", "fork", "share", "free"])
        a = int(rng.integers(0, max_seqs))
        if kind == "add":
            ops.append(("add", a))
        elif kind == "append":
            ops.append(("append", a, int(rng.integers(1, max_append + 1))))
        elif kind == "fork":
            ops.append(("fork", a, int(rng.integers(0, max_seqs))))
        elif kind == "share":
            ops.append(("share", a, int(rng.integers(0, max_seqs)), int(rng.integers(0, 8))))
        else:
            ops.append(("free", a))
    return ops
