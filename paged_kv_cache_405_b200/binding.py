"""ctypes binding for ``libpagedkv.so`` -- argument marshalling only.

Every function here forwards to the C call of the same name (``pkv_`` prefix
dropped) declared in ``include/pagedkv.h``; shapes are read off the torch
tensors, pointers passed as integers, and a non-OK status raises
``PagedKVError``.  All computation happens in the library's CUDA kernels and
its C++ allocator.  There is no fallback: if the library is missing, importing
this module fails; device calls demand CUDA tensors.
"""
from __future__ import annotations

import ctypes
import functools
import os
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# PKV_LIBRARY may name another build of the same library (e.g. other launch shapes).
LIB_PATH = os.environ.get("PKV_LIBRARY") or os.path.join(_HERE, "libpagedkv.so")

OK, INVALID, NO_FREE_BLOCK, CUDA_ERROR, UNSUPPORTED, DEVICE_CHECK = range(6)
DEVERR_BLOCK_ID, DEVERR_SLOT, DEVERR_CONTEXT, DEVERR_TIMEOUT, DEVERR_GROUP, DEVERR_SPLIT = 1, 2, 4, 8, 16, 32
_DTYPE = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}
FP8_E4M3 = 3  # pool element type of the _fp8 calls (uint8 tensors of E4M3 codes)

# Every symbol include/pagedkv.h declares.
EXPORTS = [
    "pkv_kv_append", "pkv_attention_workspace_bytes", "pkv_attention_partition_size",
    "pkv_paged_attention_decode", "pkv_paged_attention_decode_static", "pkv_paged_attention_decode_shared",
    "pkv_attention_shared_workspace_bytes", "pkv_find_shared_prefix_groups", "pkv_paged_attention_chunk",
    "pkv_attention_chunk_workspace_bytes", "pkv_kv_append_fp8", "pkv_paged_attention_decode_fp8", "pkv_block_copy", "pkv_device_error", "pkv_launch_count",
    "pkv_alloc_create", "pkv_alloc_destroy", "pkv_seq_add", "pkv_seq_share_prefix", "pkv_seq_fork",
    "pkv_alloc_set_prefix_caching", "pkv_seq_add_with_prompt", "pkv_seq_append_tokens", "pkv_prefix_cache_stats",
    "pkv_seq_append_slots", "pkv_seq_append_slots_batch", "pkv_seq_block_tables_batch", "pkv_seq_lens_batch", "pkv_seq_free", "pkv_seq_block_table", "pkv_alloc_stats",
    "pkv_block_refcount", "pkv_status_str", "pkv_last_error", "pkv_step_from_host",
]

# pkv_step_kind
STEP_DECODE, STEP_DECODE_SHARED, STEP_DECODE_FP8, STEP_CHUNK = range(4)


class PkvCopy(ctypes.Structure):
    """pkv_copy: one asynchronous copy of pkv_step_from_host."""
    _fields_ = [("dst", ctypes.c_void_p), ("src", ctypes.c_void_p), ("bytes", ctypes.c_size_t)]


class PkvStep(ctypes.Structure):
    """pkv_step, field for field (``in_`` is the header's ``in``)."""
    _fields_ = [
        ("struct_size", ctypes.c_size_t), ("kind", ctypes.c_int),
        ("in_", ctypes.POINTER(PkvCopy)), ("n_in", ctypes.c_int),
        ("out", ctypes.POINTER(PkvCopy)), ("n_out", ctypes.c_int),
        ("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p),
        ("num_blocks", ctypes.c_int), ("num_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
        ("block_size", ctypes.c_int), ("dtype", ctypes.c_int), ("k_scale", ctypes.c_float),
        ("v_scale", ctypes.c_float),
        ("pairs", ctypes.c_void_p), ("num_pairs", ctypes.c_int),
        ("k_new", ctypes.c_void_p), ("v_new", ctypes.c_void_p), ("slot_mapping", ctypes.c_void_p),
        ("num_tokens", ctypes.c_int),
        ("attn_out", ctypes.c_void_p), ("q", ctypes.c_void_p), ("block_tables", ctypes.c_void_p),
        ("max_blocks_per_seq", ctypes.c_int), ("context_lens", ctypes.c_void_p),
        ("num_seqs", ctypes.c_int), ("num_q_heads", ctypes.c_int), ("scale", ctypes.c_float),
        ("partition_size", ctypes.c_int), ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("group_first", ctypes.c_void_p), ("group_shared", ctypes.c_void_p), ("num_groups", ctypes.c_int),
        ("max_group_size", ctypes.c_int), ("max_shared_len", ctypes.c_int),
        ("query_start", ctypes.c_void_p), ("max_query_len", ctypes.c_int),
        ("copy_stream", ctypes.c_void_p), ("inputs_free", ctypes.c_void_p), ("inputs_ready", ctypes.c_void_p),
        ("out_stream", ctypes.c_void_p), ("outputs_done", ctypes.c_void_p),
    ]


class PagedKVError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__("%s (status %d)" % (msg, status))
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("libpagedkv.so is not built; run `python paged_kv_cache_405_b200/build.py` "
                          "or __graft_entry__.build()")
    lib = ctypes.CDLL(LIB_PATH)
    c_int, c_i64, c_vp, c_sz = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t
    sig = {
        "pkv_kv_append": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_int, c_int, c_int, c_int, c_int, c_vp]),
        "pkv_attention_workspace_bytes": (c_sz, [c_int, c_int, c_int, c_int, c_int]),
        "pkv_attention_partition_size": (c_int, [c_int, c_int, c_int, c_int, c_int, c_int]),
        "pkv_paged_attention_decode": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_vp, c_int, c_int, c_int,
                                               c_int, c_int, c_int, ctypes.c_float, c_int, c_vp, c_sz, c_int,
                                               c_vp]),
        "pkv_paged_attention_decode_static": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_vp, c_int, c_int,
                                                      c_int, c_int, c_int, c_int, ctypes.c_float, c_int, c_int,
                                                      c_vp]),
        "pkv_paged_attention_decode_shared": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_vp, c_int, c_int,
                                                      c_int, c_int, c_int, c_int, ctypes.c_float, c_int, c_vp,
                                                      c_vp, c_int, c_int, c_int, c_vp, c_sz, c_int, c_vp]),
        "pkv_attention_shared_workspace_bytes": (c_sz, [c_int, c_int, c_int, c_int, c_int]),
        "pkv_paged_attention_chunk": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_vp, c_vp, c_int, c_int, c_int,
                                              c_int, c_int, c_int, c_int, c_int, ctypes.c_float, c_int, c_vp, c_sz,
                                              c_int, c_vp]),
        "pkv_attention_chunk_workspace_bytes": (c_sz, [c_int, c_int, c_int, c_int, c_int]),
        "pkv_kv_append_fp8": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_int, c_int, c_int, c_int, c_int,
                                      ctypes.c_float, ctypes.c_float, c_vp]),
        "pkv_paged_attention_decode_fp8": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_vp, c_int, c_int, c_int,
                                                   c_int, c_int, c_int, ctypes.c_float, ctypes.c_float,
                                                   ctypes.c_float, c_int, c_vp, c_sz, c_int, c_vp]),
        "pkv_find_shared_prefix_groups": (c_int, [c_vp, c_vp, c_int, c_int, c_int, c_int, c_vp, c_vp, c_int,
                                                  ctypes.POINTER(c_int)]),
        "pkv_block_copy": (c_int, [c_vp, c_vp, c_vp, c_int, c_int, c_int, c_int, c_int, c_int, c_vp]),
        "pkv_device_error": (c_int, [c_vp, ctypes.POINTER(ctypes.c_uint32)]),
        "pkv_launch_count": (ctypes.c_uint64, []),
        "pkv_alloc_create": (c_vp, [c_int, c_int, c_vp]),
        "pkv_alloc_destroy": (None, [c_vp]),
        "pkv_seq_add": (c_int, [c_vp, c_i64]),
        "pkv_seq_share_prefix": (c_int, [c_vp, c_i64, c_vp, c_int, c_int]),
        "pkv_seq_fork": (c_int, [c_vp, c_i64, c_i64]),
        "pkv_seq_append_slots": (c_int, [c_vp, c_i64, c_int, c_vp, c_vp, c_int, ctypes.POINTER(c_int)]),
        "pkv_seq_append_slots_batch": (c_int, [c_vp, c_vp, c_int, c_vp, c_vp, c_int, ctypes.POINTER(c_int)]),
        "pkv_seq_block_tables_batch": (c_int, [c_vp, c_vp, c_int, c_vp, c_int, c_vp]),
        "pkv_seq_lens_batch": (c_int, [c_vp, c_vp, c_int, c_vp]),
        "pkv_seq_free": (c_int, [c_vp, c_i64]),
        "pkv_alloc_set_prefix_caching": (c_int, [c_vp, c_int]),
        "pkv_seq_add_with_prompt": (c_int, [c_vp, c_i64, c_vp, c_int, c_vp, ctypes.POINTER(c_int)]),
        "pkv_seq_append_tokens": (c_int, [c_vp, c_i64, c_vp, c_int, c_vp, c_vp, c_int, ctypes.POINTER(c_int)]),
        "pkv_prefix_cache_stats": (c_int, [c_vp, ctypes.POINTER(c_i64), ctypes.POINTER(c_i64),
                                           ctypes.POINTER(c_int), ctypes.POINTER(c_int), ctypes.POINTER(c_i64)]),
        "pkv_seq_block_table": (c_int, [c_vp, c_i64, c_vp, c_int, ctypes.POINTER(c_int),
                                        ctypes.POINTER(c_i64)]),
        "pkv_alloc_stats": (c_int, [c_vp, ctypes.POINTER(c_int), ctypes.POINTER(c_int),
                                    ctypes.POINTER(c_i64), ctypes.POINTER(c_i64)]),
        "pkv_block_refcount": (c_int, [c_vp, c_int]),
        "pkv_status_str": (ctypes.c_char_p, [c_int]),
        "pkv_step_from_host": (c_int, [ctypes.POINTER(PkvStep), c_vp]),
        "pkv_last_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


def _check(status: int):
    if status != OK:
        raise PagedKVError(status, lib.pkv_last_error().decode() or lib.pkv_status_str(status).decode())


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: torch.Tensor, name: str) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t.data_ptr()


def _dt(t: torch.Tensor) -> int:
    if t.dtype not in _DTYPE:
        raise TypeError("element type must be float32, bfloat16 or float16")
    return _DTYPE[t.dtype]


# The C calls see pointers and the sizes passed next to them, not the tensors:
# these checks make the sizes read off one tensor hold for the others, so that
# no call reads or writes past a caller's buffer.
def _cuda(**tensors) -> None:
    for name, t in tensors.items():
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise TypeError("%s must be a CUDA tensor" % name)


def _check_pools(k_pool, v_pool) -> None:
    if k_pool.dim() != 4:
        raise ValueError("pools must be [num_blocks, num_kv_heads, block_size, head_dim]")
    if v_pool.shape != k_pool.shape or v_pool.dtype != k_pool.dtype:
        raise ValueError("k_pool and v_pool must have the same shape and element type")


def _check_new(k_new, v_new, k_pool, slot_mapping, pool_type: bool) -> None:
    """New K/V [T, num_kv_heads, head_dim] of the pools, one slot per token;
    pool_type: in the pools' element type (the FP8 append converts)."""
    if k_new.dim() != 3 or tuple(k_new.shape[1:]) != (k_pool.shape[1], k_pool.shape[3]):
        raise ValueError("new K/V must be [T, num_kv_heads, head_dim] of the pools")
    if v_new.shape != k_new.shape or v_new.dtype != k_new.dtype:
        raise ValueError("k_new and v_new must have the same shape and element type")
    if pool_type and k_new.dtype != k_pool.dtype:
        raise TypeError("new K/V must have the pools' element type")
    if slot_mapping.numel() < k_new.shape[0]:
        raise ValueError("slot_mapping needs one entry per new token")


def _check_attention(out, q, k_pool, block_tables, context_lens, rows: int, pool_type: bool) -> None:
    """out like q [rows of q, num_q_heads, head_dim]; tables and lengths for
    ``rows`` sequences; pool_type: q in the pools' element type (not FP8)."""
    if q.dim() != 3 or out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("out must have the shape and element type of q [rows, num_q_heads, head_dim]")
    if q.shape[2] != k_pool.shape[3]:
        raise ValueError("q's head_dim differs from the pools'")
    if pool_type and q.dtype != k_pool.dtype:
        raise TypeError("q, out and the pools must share one element type")
    if block_tables.dim() != 2 or block_tables.shape[0] < rows:
        raise ValueError("block_tables must be [num_seqs, max_blocks_per_seq]")
    if context_lens.numel() < rows:
        raise ValueError("context_lens needs one entry per sequence")


# ------------------------------------------------------------------ NVTX ranges
_NVTX = False


def set_nvtx(on: bool) -> None:
    """Mark every device call with an NVTX range named after its C entry point
    (``pkv_kv_append``, ``pkv_paged_attention_decode`` ...), for ``ncu --nvtx``
    filters and timeline tools.  Off by default."""
    global _NVTX
    _NVTX = bool(on)


def _ranged(cname: str):
    def wrap(fn):
        @functools.wraps(fn)
        def call(*args, **kwargs):
            if not _NVTX:
                return fn(*args, **kwargs)
            torch.cuda.nvtx.range_push(cname)
            try:
                return fn(*args, **kwargs)
            finally:
                torch.cuda.nvtx.range_pop()
        return call
    return wrap


def raw_call(cname: str, *args) -> None:
    """Call the C entry point ``cname`` with arguments already marshalled
    (device pointers as ints, sizes, a stream handle) and raise on a non-OK
    status.  For callers that checked their buffers against the sizes once,
    up front (``DecodeSession``'s host-buffer steps reuse buffers it made
    itself); the C call still does its own argument checks."""
    f = getattr(lib, cname)
    if not _NVTX:
        _check(f(*args))
        return
    torch.cuda.nvtx.range_push(cname)
    try:
        _check(f(*args))
    finally:
        torch.cuda.nvtx.range_pop()


# ------------------------------------------------------------------ device calls
@_ranged("pkv_kv_append")
def kv_append(k_new, v_new, k_pool, v_pool, slot_mapping, stream=None) -> None:
    """Write token i's K/V ``[T, Hkv, D]`` into pool slot ``slot_mapping[i]`` (int64; < 0 skips)."""
    _cuda(k_new=k_new, v_new=v_new, k_pool=k_pool, v_pool=v_pool, slot_mapping=slot_mapping)
    _check_pools(k_pool, v_pool)
    NB, Hkv, bs, D = k_pool.shape
    T = k_new.shape[0]
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    _check_new(k_new, v_new, k_pool, slot_mapping, pool_type=True)
    _check(lib.pkv_kv_append(_dev(k_new, "k_new"), _dev(v_new, "v_new"), _dev(k_pool, "k_pool"),
                             _dev(v_pool, "v_pool"), _dev(slot_mapping, "slot_mapping"), T, NB, Hkv, D, bs,
                             _dt(k_pool), _stream(stream)))


def attention_workspace_bytes(num_seqs: int, num_q_heads: int, head_dim: int, max_context_len: int,
                              partition_size: int = 0) -> int:
    return int(lib.pkv_attention_workspace_bytes(num_seqs, num_q_heads, head_dim, max_context_len,
                                                 partition_size))


def attention_partition_size(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                             partition_size=0) -> int:
    return int(lib.pkv_attention_partition_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                max_context_len, partition_size))


def workspace_for(q, block_tables, block_size, partition_size=0) -> torch.Tensor:
    """Allocate (via torch) a workspace big enough for a decode call with these inputs."""
    S, Hq, D = q.shape
    n = attention_workspace_bytes(S, Hq, D, block_tables.shape[1] * block_size, partition_size)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)


@_ranged("pkv_paged_attention_decode")
def paged_attention_decode(out, q, k_pool, v_pool, block_tables, context_lens, scale: float = 0.0,
                           partition_size: int = 0, workspace: Optional[torch.Tensor] = None,
                           stream=None) -> torch.Tensor:
    """Decode attention: ``out[s, h] = softmax(scale q K^T) V`` over ``context_lens[s]`` cached tokens."""
    _cuda(out=out, q=q, k_pool=k_pool, v_pool=v_pool, block_tables=block_tables, context_lens=context_lens)
    _check_pools(k_pool, v_pool)
    S, Hq, D = q.shape
    NB, Hkv, bs, _ = k_pool.shape
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    _check_attention(out, q, k_pool, block_tables, context_lens, S, pool_type=True)
    maxB = block_tables.shape[1]
    if workspace is None:
        workspace = workspace_for(q, block_tables, bs, partition_size)
    ws_ptr = _dev(workspace, "workspace")
    _check(lib.pkv_paged_attention_decode(
        _dev(out, "out"), _dev(q, "q"), _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"),
        _dev(block_tables, "block_tables"), maxB, _dev(context_lens, "context_lens"), S, Hq, Hkv, D, bs, NB,
        float(scale), int(partition_size), ws_ptr, workspace.numel() * workspace.element_size(), _dt(q),
        _stream(stream)))
    return out


@_ranged("pkv_paged_attention_decode_static")
def paged_attention_decode_static(out, q, k_pool, v_pool, block_tables, context_lens, scale: float = 0.0,
                                  partition_size: int = 0, stream=None) -> torch.Tensor:
    """Decode attention that allocates nothing: the split-K scratch is a fixed
    64 MiB buffer inside the library (one per GPU), for callers that cannot
    allocate device memory.  Calls on one device share that buffer, so calls
    that overlap on the GPU must not be issued; oversized calls raise."""
    _cuda(out=out, q=q, k_pool=k_pool, v_pool=v_pool, block_tables=block_tables, context_lens=context_lens)
    _check_pools(k_pool, v_pool)
    S, Hq, D = q.shape
    NB, Hkv, bs, _ = k_pool.shape
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    _check_attention(out, q, k_pool, block_tables, context_lens, S, pool_type=True)
    _check(lib.pkv_paged_attention_decode_static(
        _dev(out, "out"), _dev(q, "q"), _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"),
        _dev(block_tables, "block_tables"), block_tables.shape[1], _dev(context_lens, "context_lens"), S, Hq, Hkv,
        D, bs, NB, float(scale), int(partition_size), _dt(q), _stream(stream)))
    return out


def attention_shared_workspace_bytes(num_seqs: int, num_q_heads: int, head_dim: int, max_context_len: int,
                                     partition_size: int = 0) -> int:
    return int(lib.pkv_attention_shared_workspace_bytes(num_seqs, num_q_heads, head_dim, max_context_len,
                                                        partition_size))


def find_shared_prefix_groups(block_tables: np.ndarray, context_lens: np.ndarray, block_size: int,
                              min_group_size: int = 4):
    """Runs of consecutive sequences whose tables start with the same blocks.
    Returns (group_first int32 [n+1], group_shared int32 [n]) -- n runs, gaps
    between groups included with shared length 0."""
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    S = bt.shape[0]
    first = np.zeros(S + 1, dtype=np.int32)
    shared = np.zeros(max(S, 1), dtype=np.int32)
    ng = ctypes.c_int(0)
    _check(lib.pkv_find_shared_prefix_groups(bt.ctypes.data, lens.ctypes.data, S, bt.shape[1], block_size,
                                             min_group_size, first.ctypes.data, shared.ctypes.data, S,
                                             ctypes.byref(ng)))
    n = ng.value
    return first[:n + 1] if n else first[:0], shared[:n]


@_ranged("pkv_paged_attention_decode_shared")
def paged_attention_decode_shared(out, q, k_pool, v_pool, block_tables, context_lens, group_first, group_shared,
                                  max_group_size: int, max_shared_len: int, scale: float = 0.0,
                                  partition_size: int = 0, workspace: Optional[torch.Tensor] = None,
                                  stream=None) -> torch.Tensor:
    """Decode attention with shared-prefix groups (device int32 group_first [n+1], group_shared [n];
    host bounds max_group_size and max_shared_len)."""
    _cuda(out=out, q=q, k_pool=k_pool, v_pool=v_pool, block_tables=block_tables, context_lens=context_lens,
          group_first=group_first, group_shared=group_shared)
    _check_pools(k_pool, v_pool)
    S, Hq, D = q.shape
    NB, Hkv, bs, _ = k_pool.shape
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    _check_attention(out, q, k_pool, block_tables, context_lens, S, pool_type=True)
    n = group_shared.numel()
    if n and group_first.numel() < n + 1:
        raise ValueError("group_first needs num_groups + 1 entries")
    maxB = block_tables.shape[1]
    if workspace is None:
        nb = attention_shared_workspace_bytes(S, Hq, D, maxB * bs, partition_size)
        workspace = torch.empty(max(nb, 256), dtype=torch.uint8, device=q.device)
    _check(lib.pkv_paged_attention_decode_shared(
        _dev(out, "out"), _dev(q, "q"), _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"),
        _dev(block_tables, "block_tables"), maxB, _dev(context_lens, "context_lens"), S, Hq, Hkv, D, bs, NB,
        float(scale), int(partition_size), _dev(group_first, "group_first") if n else None,
        _dev(group_shared, "group_shared") if n else None, n, int(max_group_size), int(max_shared_len),
        _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _dt(q), _stream(stream)))
    return out


def attention_chunk_workspace_bytes(num_tokens: int, num_q_heads: int, head_dim: int, max_context_len: int,
                                    partition_size: int = 0) -> int:
    return int(lib.pkv_attention_chunk_workspace_bytes(num_tokens, num_q_heads, head_dim, max_context_len,
                                                       partition_size))


@_ranged("pkv_paged_attention_chunk")
def paged_attention_chunk(out, q, k_pool, v_pool, block_tables, context_lens, query_start, max_query_len: int,
                          scale: float = 0.0, partition_size: int = 0, workspace: Optional[torch.Tensor] = None,
                          stream=None) -> torch.Tensor:
    """Causal attention of the last ``query_start[s+1]-query_start[s]`` tokens of each sequence."""
    _cuda(out=out, q=q, k_pool=k_pool, v_pool=v_pool, block_tables=block_tables, context_lens=context_lens,
          query_start=query_start)
    _check_pools(k_pool, v_pool)
    T, Hq, D = q.shape
    NB, Hkv, bs, _ = k_pool.shape
    for t, nm in ((block_tables, "block_tables"), (context_lens, "context_lens"), (query_start, "query_start")):
        if t.dtype != torch.int32:
            raise TypeError("%s must be int32" % nm)
    S = context_lens.numel()
    _check_attention(out, q, k_pool, block_tables, context_lens, S, pool_type=True)
    if query_start.numel() < S + 1:
        raise ValueError("query_start needs num_seqs + 1 entries")
    maxB = block_tables.shape[1]
    if workspace is None:
        nb = attention_chunk_workspace_bytes(T, Hq, D, maxB * bs, partition_size)
        workspace = torch.empty(max(nb, 256), dtype=torch.uint8, device=q.device)
    _check(lib.pkv_paged_attention_chunk(
        _dev(out, "out"), _dev(q, "q"), _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"),
        _dev(block_tables, "block_tables"), maxB, _dev(context_lens, "context_lens"),
        _dev(query_start, "query_start"), S, T, int(max_query_len), Hq, Hkv, D, bs, NB, float(scale),
        int(partition_size), _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(), _dt(q),
        _stream(stream)))
    return out


@_ranged("pkv_kv_append_fp8")
def kv_append_fp8(k_new, v_new, k_pool, v_pool, slot_mapping, k_scale: float, v_scale: float,
                  stream=None) -> None:
    """Quantize new K/V ([T, Hkv, D], f32/bf16/f16) into FP8 E4M3 pools (uint8 [NB, Hkv, bs, D])."""
    _cuda(k_new=k_new, v_new=v_new, k_pool=k_pool, v_pool=v_pool, slot_mapping=slot_mapping)
    _check_pools(k_pool, v_pool)
    NB, Hkv, bs, D = k_pool.shape
    if k_pool.dtype != torch.uint8 or v_pool.dtype != torch.uint8:
        raise TypeError("FP8 pools are uint8 tensors of E4M3 codes")
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    _check_new(k_new, v_new, k_pool, slot_mapping, pool_type=False)
    _check(lib.pkv_kv_append_fp8(_dev(k_new, "k_new"), _dev(v_new, "v_new"), _dev(k_pool, "k_pool"),
                                 _dev(v_pool, "v_pool"), _dev(slot_mapping, "slot_mapping"), k_new.shape[0], NB,
                                 Hkv, D, bs, _dt(k_new), float(k_scale), float(v_scale), _stream(stream)))


@_ranged("pkv_paged_attention_decode_fp8")
def paged_attention_decode_fp8(out, q, k_pool, v_pool, block_tables, context_lens, k_scale: float,
                               v_scale: float, scale: float = 0.0, partition_size: int = 0,
                               workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Decode attention over FP8 E4M3 pools (values = code x k_scale / x v_scale); q/out bf16 or f16."""
    _cuda(out=out, q=q, k_pool=k_pool, v_pool=v_pool, block_tables=block_tables, context_lens=context_lens)
    _check_pools(k_pool, v_pool)
    S, Hq, D = q.shape
    NB, Hkv, bs, _ = k_pool.shape
    if k_pool.dtype != torch.uint8 or v_pool.dtype != torch.uint8:
        raise TypeError("FP8 pools are uint8 tensors of E4M3 codes")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    _check_attention(out, q, k_pool, block_tables, context_lens, S, pool_type=False)
    maxB = block_tables.shape[1]
    if workspace is None:
        workspace = workspace_for(q, block_tables, bs, partition_size)
    _check(lib.pkv_paged_attention_decode_fp8(
        _dev(out, "out"), _dev(q, "q"), _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"),
        _dev(block_tables, "block_tables"), maxB, _dev(context_lens, "context_lens"), S, Hq, Hkv, D, bs, NB,
        float(scale), float(k_scale), float(v_scale), int(partition_size), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _dt(q), _stream(stream)))
    return out


@_ranged("pkv_block_copy")
def block_copy(k_pool, v_pool, pairs, stream=None) -> None:
    """Copy whole blocks ``pairs[i] = (src, dst)`` (int32 ``[n, 2]`` on the device), K and V."""
    _cuda(k_pool=k_pool, v_pool=v_pool, pairs=pairs)
    _check_pools(k_pool, v_pool)
    NB, Hkv, bs, D = k_pool.shape
    if pairs.dtype != torch.int32:
        raise TypeError("pairs must be int32")
    if pairs.numel() and (pairs.dim() != 2 or pairs.shape[1] != 2):
        raise ValueError("pairs must be [n, 2] (src, dst)")
    n = pairs.shape[0] if pairs.numel() else 0
    dt = FP8_E4M3 if k_pool.dtype == torch.uint8 else _dt(k_pool)
    _check(lib.pkv_block_copy(_dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"),
                              _dev(pairs, "pairs") if n else None, n, NB, Hkv, D, bs, dt, _stream(stream)))


def step_from_host(step: PkvStep, stream=None) -> None:
    """One whole step in one C call (see pkv_step_from_host): ``step`` is a
    filled-in ``PkvStep``; DecodeSession.launch_step builds and fills one."""
    raw_call("pkv_step_from_host", ctypes.byref(step), _stream(stream))


def device_error(stream=None) -> int:
    """Wait for the stream; return and clear the device error word (0 = clean)."""
    code = ctypes.c_uint32(0)
    st = lib.pkv_device_error(_stream(stream), ctypes.byref(code))
    if st not in (OK, DEVICE_CHECK):
        _check(st)
    return int(code.value)


def launch_count() -> int:
    return int(lib.pkv_launch_count())


# -------------------------------------------------------------- host allocator
class BlockAllocator:
    """The library's host block allocator (free pool, refcounts, block tables, COW)."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None, prefix_caching: bool = False):
        self.num_blocks = num_blocks
        self.block_size = block_size
        fo = None
        if free_order is not None:
            self._fo = np.ascontiguousarray(np.asarray(free_order, dtype=np.int32))
            fo = self._fo.ctypes.data
        h = lib.pkv_alloc_create(num_blocks, block_size, fo)
        if not h:
            raise PagedKVError(INVALID, lib.pkv_last_error().decode())
        self._h = ctypes.c_void_p(h)
        self._destroy = lib.pkv_alloc_destroy  # kept: module globals may be gone at interpreter exit
        if prefix_caching:
            _check(lib.pkv_alloc_set_prefix_caching(self._h, 1))
        self._slots = np.zeros(64, dtype=np.int64)
        self._cow = np.zeros(2, dtype=np.int32)

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            self._destroy(h)
            self._h = None

    def seq_add(self, sid: int) -> int:
        return lib.pkv_seq_add(self._h, sid)

    def seq_share_prefix(self, sid: int, blocks, ntok: int) -> int:
        b = np.ascontiguousarray(np.asarray(blocks, dtype=np.int32))
        return lib.pkv_seq_share_prefix(self._h, sid, b.ctypes.data if len(b) else None, len(b), ntok)

    def seq_fork(self, parent: int, child: int) -> int:
        return lib.pkv_seq_fork(self._h, parent, child)

    def seq_append_slots(self, sid: int, n: int):
        """Returns (status, slots list, [(src, dst)] copy-on-write pairs)."""
        if n > len(self._slots):
            self._slots = np.zeros(max(n, 2 * len(self._slots)), dtype=np.int64)
        ncow = ctypes.c_int(0)
        st = lib.pkv_seq_append_slots(self._h, sid, n, self._slots.ctypes.data, self._cow.ctypes.data, 1,
                                      ctypes.byref(ncow))
        if st != OK:
            return st, [], []
        pairs = [(int(self._cow[0]), int(self._cow[1]))] if ncow.value else []
        return st, self._slots[:n].tolist(), pairs

    def seq_append_slots_batch(self, sids):
        """One slot for each sequence id, in order.  Returns (status, slots int64 array,
        cow pairs int32 [n, 2] array)."""
        ids = np.ascontiguousarray(np.asarray(sids, dtype=np.int64))
        n = len(ids)
        slots = np.zeros(n, dtype=np.int64)
        cow = np.zeros((max(n, 1), 2), dtype=np.int32)
        ncow = ctypes.c_int(0)
        st = lib.pkv_seq_append_slots_batch(self._h, ids.ctypes.data, n, slots.ctypes.data, cow.ctypes.data,
                                            max(n, 1), ctypes.byref(ncow))
        if st != OK:
            return st, slots[:0], cow[:0]
        return st, slots, cow[:ncow.value]

    def seq_block_tables_batch(self, sids, max_blocks: int, out=None, lens_out=None):
        """Block tables (int32 [n, max_blocks], -1 padded) and lengths (int32 [n])."""
        ids = np.ascontiguousarray(np.asarray(sids, dtype=np.int64))
        n = len(ids)
        out = np.empty((n, max_blocks), dtype=np.int32) if out is None else out
        lens_out = np.empty(n, dtype=np.int32) if lens_out is None else lens_out
        st = lib.pkv_seq_block_tables_batch(self._h, ids.ctypes.data, n, out.ctypes.data, max_blocks,
                                            lens_out.ctypes.data)
        return st, out, lens_out

    def seq_lens_batch(self, sids):
        """Lengths in tokens (int64 [n]) of many sequences.  Returns (status, lengths)."""
        ids = np.ascontiguousarray(np.asarray(sids, dtype=np.int64))
        lens = np.empty(len(ids), dtype=np.int64)
        st = lib.pkv_seq_lens_batch(self._h, ids.ctypes.data, len(ids), lens.ctypes.data)
        return st, lens

    def seq_add_with_prompt(self, sid: int, tokens):
        """Returns (status, cached tokens, slots of the remaining tokens)."""
        t = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
        slots = np.zeros(max(len(t), 1), dtype=np.int64)
        nc = ctypes.c_int(0)
        st = lib.pkv_seq_add_with_prompt(self._h, sid, t.ctypes.data if len(t) else None, len(t),
                                         slots.ctypes.data, ctypes.byref(nc))
        if st != OK:
            return st, 0, []
        return st, nc.value, slots[:len(t) - nc.value].tolist()

    def seq_append_tokens(self, sid: int, tokens):
        """Returns (status, slots, [(src, dst)] copy-on-write pairs)."""
        t = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
        n = len(t)
        slots = np.zeros(max(n, 1), dtype=np.int64)
        ncow = ctypes.c_int(0)
        st = lib.pkv_seq_append_tokens(self._h, sid, t.ctypes.data if n else None, n, slots.ctypes.data,
                                       self._cow.ctypes.data, 1, ctypes.byref(ncow))
        if st != OK:
            return st, [], []
        pairs = [(int(self._cow[0]), int(self._cow[1]))] if ncow.value else []
        return st, slots[:n].tolist(), pairs

    def cache_stats(self) -> dict:
        lk, ht, ev = ctypes.c_int64(0), ctypes.c_int64(0), ctypes.c_int64(0)
        cb, eb = ctypes.c_int(0), ctypes.c_int(0)
        _check(lib.pkv_prefix_cache_stats(self._h, ctypes.byref(lk), ctypes.byref(ht), ctypes.byref(cb),
                                          ctypes.byref(eb), ctypes.byref(ev)))
        return dict(lookups=lk.value, hits=ht.value, cached_blocks=cb.value, evictable_blocks=eb.value,
                    evictions=ev.value)

    def seq_free(self, sid: int) -> int:
        return lib.pkv_seq_free(self._h, sid)

    def seq_block_table(self, sid: int):
        """Returns (status, block table list, length in tokens)."""
        n = ctypes.c_int(-1)
        ln = ctypes.c_int64(0)
        st = lib.pkv_seq_block_table(self._h, sid, None, 0, ctypes.byref(n), ctypes.byref(ln))
        if n.value < 0:          # unknown sequence
            return st, [], 0
        if n.value == 0:
            return OK, [], int(ln.value)
        buf = np.zeros(n.value, dtype=np.int32)
        st = lib.pkv_seq_block_table(self._h, sid, buf.ctypes.data, n.value, ctypes.byref(n), ctypes.byref(ln))
        if st != OK:
            return st, [], 0
        return st, buf.tolist(), int(ln.value)

    def stats(self) -> dict:
        f, u = ctypes.c_int(0), ctypes.c_int(0)
        af, cc = ctypes.c_int64(0), ctypes.c_int64(0)
        _check(lib.pkv_alloc_stats(self._h, ctypes.byref(f), ctypes.byref(u), ctypes.byref(af), ctypes.byref(cc)))
        return dict(free_blocks=f.value, used_blocks=u.value, alloc_failures=af.value, cow_copies=cc.value)

    def refcount(self, block: int) -> int:
        return lib.pkv_block_refcount(self._h, block)
