"""CPU oracle for paged decode -- TEST INFRASTRUCTURE ONLY.

Plain, slow and obviously correct.  Only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline leg may import this package; the product path
(the ``paged_kv_cache_405_b200`` package and its CUDA library) never does, and
nothing here imports the product.

Contents
--------
* ``paged_attention`` -- fp64 decode attention over the paged pool (C, see
  ``oracle.c`` for the definition and its citations).
* ``slot`` -- block-table translation of one token.
* ``kv_append`` / ``block_copy`` -- the two byte-moving operations, on CPU
  tensors, as plain indexing.
* ``Allocator`` (``allocator.py``) -- free pool, refcounts, block tables,
  sharing and copy-on-write.
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np
import torch

from . import build as _build
from .allocator import INVALID, NO_FREE_BLOCK, OK, Allocator  # noqa: F401

_DT = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}
_lib = None


def _load():
    global _lib
    if _lib is None:
        # ORACLE_LIBRARY may name another build of oracle.c (the tests build
        # copies with planted mistakes to show that the pins catch them).
        lib = ctypes.CDLL(os.environ.get("ORACLE_LIBRARY") or _build.build())
        lib.oracle_paged_attention.restype = ctypes.c_int
        lib.oracle_paged_attention.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int]
        lib.oracle_slot.restype = ctypes.c_int64
        lib.oracle_slot.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int64]
        lib.oracle_max_threads.restype = ctypes.c_int
        lib.oracle_paged_attention_kv.restype = ctypes.c_int
        lib.oracle_paged_attention_kv.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
            ctypes.c_double, ctypes.c_double, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int]
        lib.oracle_e4m3_table.restype = None
        lib.oracle_e4m3_table.argtypes = [ctypes.c_void_p]
        lib.oracle_paged_attention_chunk.restype = ctypes.c_int
        lib.oracle_paged_attention_chunk.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int]
        _lib = lib
    return _lib


def max_threads() -> int:
    return _load().oracle_max_threads()


def _cpu(t):
    if isinstance(t, np.ndarray):
        return torch.from_numpy(np.ascontiguousarray(t))
    return t.detach().to("cpu").contiguous()


def slot(bt_row, block_size: int, t: int) -> int:
    """Physical slot of token ``t`` given one block-table row."""
    row = np.ascontiguousarray(np.asarray(bt_row, dtype=np.int32))
    return int(_load().oracle_slot(row.ctypes.data, block_size, t))


def paged_attention(q, k_pool, v_pool, block_tables, context_lens, scale=None,
                    items=None, threads: int = 1) -> np.ndarray:
    """fp64 decode attention.

    q ``[S, Hq, D]``; pools ``[NB, Hkv, bs, D]`` (fp32/bf16/f16, same dtype);
    block_tables int32 ``[S, maxB]``; context_lens ``[S]``.  ``scale`` defaults
    to 1/sqrt(D).  ``items`` is an optional list of (s, h) pairs; the result is
    then ``[len(items), D]``, else ``[S, Hq, D]``.
    """
    q, k_pool, v_pool = _cpu(q), _cpu(k_pool), _cpu(v_pool)
    if not (q.dtype == k_pool.dtype == v_pool.dtype) or q.dtype not in _DT:
        raise TypeError("q and pools must share one of fp32/bf16/f16")
    S, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_pool.shape
    if D2 != D or tuple(v_pool.shape) != tuple(k_pool.shape):
        raise ValueError("shape mismatch")
    bt = np.ascontiguousarray(np.asarray(block_tables, dtype=np.int32))
    cl = np.ascontiguousarray(np.asarray(context_lens, dtype=np.int32))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if items is None:
        ss, hh = np.meshgrid(np.arange(S), np.arange(Hq), indexing="ij")
        its = np.stack([ss.ravel(), hh.ravel()], 1).astype(np.int32)
    else:
        its = np.asarray(items, dtype=np.int32).reshape(-1, 2)
    its_s = np.ascontiguousarray(its[:, 0])
    its_h = np.ascontiguousarray(its[:, 1])
    out = np.zeros((len(its), D), dtype=np.float64)
    rc = _load().oracle_paged_attention(
        out.ctypes.data, q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(),
        bt.ctypes.data, bt.shape[1], cl.ctypes.data, S, Hq, Hkv, D, bs, NB,
        float(scale), _DT[q.dtype], its_s.ctypes.data, its_h.ctypes.data, len(its), threads)
    if rc != 0:
        raise ValueError("oracle_paged_attention: invalid indices (status %d)" % rc)
    if items is None:
        return out.reshape(S, Hq, D)
    return out


def paged_attention_chunk(q, k_pool, v_pool, block_tables, context_lens, query_start, scale=None,
                          items=None, threads: int = 1) -> np.ndarray:
    """fp64 causal attention of a chunk of new tokens per sequence.

    q ``[T, Hq, D]``: rows ``query_start[s] .. query_start[s+1]-1`` are the
    last tokens of sequence s's ``context_lens[s]`` cached tokens; each attends
    to the cache up to and including its own position.  Returns ``[T, Hq, D]``
    or ``[len(items), D]`` for (row, head) ``items``.
    """
    q, k_pool, v_pool = _cpu(q), _cpu(k_pool), _cpu(v_pool)
    if not (q.dtype == k_pool.dtype == v_pool.dtype) or q.dtype not in _DT:
        raise TypeError("q and pools must share one of fp32/bf16/f16")
    T, Hq, D = q.shape
    NB, Hkv, bs, _ = k_pool.shape
    bt = np.ascontiguousarray(np.asarray(block_tables, dtype=np.int32))
    cl = np.ascontiguousarray(np.asarray(context_lens, dtype=np.int32))
    qs = np.ascontiguousarray(np.asarray(query_start, dtype=np.int32))
    S = len(cl)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if items is None:
        tt, hh = np.meshgrid(np.arange(T), np.arange(Hq), indexing="ij")
        its = np.stack([tt.ravel(), hh.ravel()], 1).astype(np.int32)
    else:
        its = np.asarray(items, dtype=np.int32).reshape(-1, 2)
    it_t = np.ascontiguousarray(its[:, 0])
    it_h = np.ascontiguousarray(its[:, 1])
    out = np.zeros((len(its), D), dtype=np.float64)
    rc = _load().oracle_paged_attention_chunk(
        out.ctypes.data, q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(), bt.ctypes.data, bt.shape[1],
        cl.ctypes.data, qs.ctypes.data, S, T, Hq, Hkv, D, bs, NB, float(scale), _DT[q.dtype],
        it_t.ctypes.data, it_h.ctypes.data, len(its), threads)
    if rc != 0:
        raise ValueError("oracle_paged_attention_chunk: invalid indices (status %d)" % rc)
    return out.reshape(T, Hq, D) if items is None else out


# ----------------------------------------------------------------- FP8 E4M3 KV
E4M3_MAX = 448.0


def e4m3_table() -> np.ndarray:
    """Value of each of the 256 E4M3 codes (NaN for the two NaN codes)."""
    out = np.zeros(256, dtype=np.float64)
    _load().oracle_e4m3_table(out.ctypes.data)
    return out


def quantize_e4m3(x, scale: float) -> np.ndarray:
    """FP8 E4M3 codes of x / scale, computed as x * (1/scale) in fp32 (the
    inverse itself rounded to fp32), rounded to nearest (ties to even) and
    saturated to +-448; NaN stays NaN.  Returns uint8 codes."""
    xf = np.asarray(_cpu(x).float().numpy(), dtype=np.float32)
    inv = np.float32(1.0) / np.float32(scale)
    y = (xf * inv).astype(np.float32).astype(np.float64).ravel()
    table = e4m3_table()
    finite = np.arange(256)[np.isfinite(table) & (table >= 0)]           # non-negative codes, ascending
    vals = table[finite]
    order = np.argsort(vals, kind="stable")
    finite, vals = finite[order], vals[order]
    keep = np.concatenate([[True], np.diff(vals) > 0])                    # +0 only (drop duplicates)
    finite, vals = finite[keep], vals[keep]
    a = np.minimum(np.abs(y), E4M3_MAX)
    hi = np.searchsorted(vals, a, side="left").clip(0, len(vals) - 1)
    lo = (hi - 1).clip(0, len(vals) - 1)
    dl, dh = np.abs(a - vals[lo]), np.abs(vals[hi] - a)
    even_hi = (finite[hi] & 1) == 0
    pick = np.where(dl < dh, lo, np.where(dh < dl, hi, np.where(even_hi, hi, lo)))
    code = finite[pick].astype(np.uint8)
    code = np.where(np.signbit(y), code | 0x80, code).astype(np.uint8)   # rounding keeps the sign (-0 too)
    code = np.where(np.isnan(y), np.uint8(0x7F), code)
    return code.reshape(np.shape(xf))


def paged_attention_kv(q, k_codes, v_codes, k_scale: float, v_scale: float, block_tables, context_lens,
                       scale=None, items=None, threads: int = 1) -> np.ndarray:
    """fp64 decode attention over FP8 E4M3 pools (uint8 codes, values = code
    value x k_scale / v_scale); q in fp32/bf16/f16."""
    q = _cpu(q)
    kc = np.ascontiguousarray(np.asarray(k_codes.cpu() if isinstance(k_codes, torch.Tensor) else k_codes,
                                         dtype=np.uint8))
    vc = np.ascontiguousarray(np.asarray(v_codes.cpu() if isinstance(v_codes, torch.Tensor) else v_codes,
                                         dtype=np.uint8))
    S, Hq, D = q.shape
    NB, Hkv, bs, _ = kc.shape
    bt = np.ascontiguousarray(np.asarray(block_tables, dtype=np.int32))
    cl = np.ascontiguousarray(np.asarray(context_lens, dtype=np.int32))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if items is None:
        ss, hh = np.meshgrid(np.arange(S), np.arange(Hq), indexing="ij")
        its = np.stack([ss.ravel(), hh.ravel()], 1).astype(np.int32)
    else:
        its = np.asarray(items, dtype=np.int32).reshape(-1, 2)
    its_s, its_h = np.ascontiguousarray(its[:, 0]), np.ascontiguousarray(its[:, 1])
    out = np.zeros((len(its), D), dtype=np.float64)
    rc = _load().oracle_paged_attention_kv(
        out.ctypes.data, q.data_ptr(), _DT[q.dtype], kc.ctypes.data, vc.ctypes.data, 3, float(np.float32(k_scale)),
        float(np.float32(v_scale)), bt.ctypes.data, bt.shape[1], cl.ctypes.data, S, Hq, Hkv, D, bs, NB,
        float(scale), its_s.ctypes.data, its_h.ctypes.data, len(its), threads)
    if rc != 0:
        raise ValueError("oracle_paged_attention_kv: invalid indices (status %d)" % rc)
    return out.reshape(S, Hq, D) if items is None else out


def kv_append_fp8(k_codes: np.ndarray, v_codes: np.ndarray, k_new, v_new, k_scale: float, v_scale: float,
                  slot_mapping) -> None:
    """Quantize each new token's K and V (quantize_e4m3) into its slot of the
    uint8 code pools, in place; a negative slot means no write."""
    bs = k_codes.shape[2]
    kq = quantize_e4m3(k_new, k_scale)
    vq = quantize_e4m3(v_new, v_scale)
    for i, sl in enumerate(np.asarray(slot_mapping, dtype=np.int64).tolist()):
        if sl < 0:
            continue
        blk, off = divmod(sl, bs)
        k_codes[blk, :, off, :] = kq[i]
        v_codes[blk, :, off, :] = vq[i]


def kv_append(k_pool: torch.Tensor, v_pool: torch.Tensor, k_new, v_new, slot_mapping) -> None:
    """Write each new token's K and V (all kv heads) into its slot, in place.

    Token i goes to block ``slot // bs`` at offset ``slot % bs``; a negative
    slot means "no write" (aiknowledge.cn 2.2.3: the new token lands in the
    sequence's last block; openeuler.csdn.net explainer 2.2: each step caches
    one new K/V).  Slots must be distinct.
    """
    bs = k_pool.shape[2]
    sm = np.asarray(slot_mapping, dtype=np.int64)
    valid = sm[sm >= 0]
    if len(np.unique(valid)) != len(valid):
        raise ValueError("duplicate slots")
    k_new, v_new = _cpu(k_new), _cpu(v_new)
    for i, sl in enumerate(sm.tolist()):
        if sl < 0:
            continue
        blk, off = divmod(sl, bs)
        k_pool[blk, :, off, :] = k_new[i]
        v_pool[blk, :, off, :] = v_new[i]


def block_copy(k_pool: torch.Tensor, v_pool: torch.Tensor, pairs) -> None:
    """Copy whole blocks (all kv heads, all offsets) src -> dst, as if at once.

    Copy-on-write copies only the block being written (openeuler.csdn.net
    explainer 6.2).  No destination may also be a source.
    """
    pr = np.asarray(pairs, dtype=np.int64).reshape(-1, 2)
    if len(pr) == 0:
        return
    src, dst = pr[:, 0].tolist(), pr[:, 1].tolist()
    if set(src) & set(dst) or len(set(dst)) != len(dst):
        raise ValueError("overlapping copy pairs")
    ks = k_pool[src].clone()
    vs = v_pool[src].clone()
    k_pool[dst] = ks
    v_pool[dst] = vs
