"""One decode step over a batch of sequences, end to end.

A step, per the pages' description of paged decoding: each running sequence
asks the block allocator for the slot of its next token (a fresh block only
when its last block is full; a private copy of a shared, partly filled last
block first -- openeuler.csdn.net PagedAttention explainer 4.3 and 6.2;
aiknowledge.cn "2.2 PagedAttention 与 KV Cache 分页管理" 2.2.3); the copies
are made (``block_copy``); the new K/V are written (``kv_append``); and every
sequence's query attends to its cached tokens through its block table
(``paged_attention_decode``).

``DecodeSession`` keeps the host side (allocator, block tables as a pinned
host array) and issues the three device calls on one stream.  ``plan`` does
the host work of a step and returns its device inputs; ``launch`` issues the
kernels for a planned step; ``step`` does both, with the host<->device copies a
serving loop makes every step (inputs in, attention output out).
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np
import torch

from . import binding as B


@dataclass
class StepPlan:
    seq_ids: list              # sequences whose query attends this step (rows of q/out)
    slot_mapping: np.ndarray   # int64 [T] slots of the tokens written this step
    cow_pairs: np.ndarray      # int32 [n, 2] blocks to copy before writing
    lens: np.ndarray           # int32 [len(seq_ids)] context after the write
    block_tables: np.ndarray   # int32 [len(seq_ids), max_blocks]
    group_first: np.ndarray = None   # int32 [g + 1] shared-prefix runs (see find_shared_prefix_groups)
    group_shared: np.ndarray = None  # int32 [g]
    max_group_size: int = 0
    max_shared_len: int = 0

    @property
    def has_groups(self) -> bool:
        return self.group_shared is not None and bool((self.group_shared > 0).any())


@dataclass
class ChunkPlan:
    seq_ids: list
    slot_mapping: np.ndarray   # int64 [T] slots of the new tokens, sequence by sequence
    cow_pairs: np.ndarray      # int32 [n, 2]
    lens: np.ndarray           # int32 [S] context after the write
    block_tables: np.ndarray   # int32 [S, max_blocks]
    query_start: np.ndarray    # int32 [S + 1]
    max_query_len: int


@dataclass
class DevicePlan:
    slot_mapping: torch.Tensor
    cow_pairs: torch.Tensor
    lens: torch.Tensor
    block_tables: torch.Tensor
    n_cow: int
    group_first: Optional[torch.Tensor] = None
    group_shared: Optional[torch.Tensor] = None
    max_group_size: int = 0
    max_shared_len: int = 0


class DecodeSession:
    def __init__(self, k_pool: torch.Tensor, v_pool: torch.Tensor, num_q_heads: int, max_blocks_per_seq: int,
                 free_order=None, partition_size: int = 0, max_batch: int = 0, share_prefixes: bool = True,
                 min_group_size: int = 4, kv_scales=None, prefix_caching: bool = False,
                 overlap_input_copies: bool = True, overlap_output_copies: bool = False):
        """Pools of a 16-bit/fp32 type, or uint8 FP8 E4M3 codes with kv_scales = (k_scale, v_scale).
        prefix_caching: full prompt blocks registered by ``add_prompt`` are
        reused by later prompts with the same leading tokens.
        overlap_input_copies: ``launch_step`` sends a step's inputs on a copy
        stream of the session's own, so that they cross while the previous
        step's kernels still run (the kernels wait for them); off, they go on
        the caller's stream ahead of the kernels.
        overlap_output_copies (needs overlap_input_copies): ``launch_step``
        copies a step's output back on a second stream of the session's own
        after the kernels, so that the next step's kernels need not wait for
        it; the caller then learns that the output has arrived only from the
        ``out_ready`` event it passes to ``launch_step``, not from its
        stream."""
        self.k_pool, self.v_pool = k_pool, v_pool
        self.fp8 = k_pool.dtype == torch.uint8
        if self.fp8 and kv_scales is None:
            raise ValueError("FP8 pools need kv_scales")
        self.kv_scales = kv_scales
        self.num_blocks, self.num_kv_heads, self.block_size, self.head_dim = k_pool.shape
        self.num_q_heads = num_q_heads
        self.max_blocks = max_blocks_per_seq
        self.partition_size = partition_size
        self.alloc = B.BlockAllocator(self.num_blocks, self.block_size, free_order, prefix_caching=prefix_caching)
        self.device = k_pool.device
        # Runs of sequences sharing leading blocks go through the shared-prefix
        # pass (16-bit pools only: it runs on tensor cores).
        self.share_prefixes = share_prefixes and k_pool.dtype not in (torch.float32, torch.uint8)
        self.min_group_size = min_group_size
        n = max(max_batch, 1)
        max_len = max_blocks_per_seq * self.block_size
        ws = B.attention_workspace_bytes(n, num_q_heads, self.head_dim, max_len, partition_size)
        if self.share_prefixes:
            ws = max(ws, B.attention_shared_workspace_bytes(n, num_q_heads, self.head_dim, max_len, partition_size))
        self.workspace = torch.empty(max(256, ws), dtype=torch.uint8, device=self.device)
        self._pinned = {}
        self._layouts = {}      # host-buffer steps: staging per layout of the step's arrays
        if overlap_output_copies and not overlap_input_copies:
            raise ValueError("overlap_output_copies needs overlap_input_copies")
        self.overlap_input_copies = overlap_input_copies
        self.overlap_output_copies = overlap_output_copies
        self._copy_stream = None
        self._out_stream = None

    # ------------------------------------------------------------ host side
    def add(self, sid: int, num_tokens: int = 0, shared_prefix: Optional[Sequence[int]] = None,
            prefix_tokens: int = 0, stream=None) -> list:
        """Register a sequence; map a shared prefix onto existing blocks, then
        reserve slots for ``num_tokens`` more tokens.  Returns their slots.

        A prefix that ends part-way through a block leaves that block shared
        and partly filled: the first reserved slot then lies in a private copy
        of it, which this call makes (``block_copy`` on ``stream``) before it
        returns, so the caller's ``kv_append`` to the returned slots must follow
        on the same stream.  If any step fails the sequence is not registered."""
        self._ok(self.alloc.seq_add(sid))
        try:
            if shared_prefix is not None:
                self._ok(self.alloc.seq_share_prefix(sid, shared_prefix, prefix_tokens))
            if not num_tokens:
                return []
            st, slots, cow = self.alloc.seq_append_slots(sid, num_tokens)
            self._ok(st)
        except Exception:
            self.alloc.seq_free(sid)
            raise
        if cow:
            s = torch.cuda.current_stream() if stream is None else stream
            with torch.cuda.stream(s):
                pairs = torch.tensor(cow, dtype=torch.int32).to(self.device)
                B.block_copy(self.k_pool, self.v_pool, pairs, stream=s)
        return slots

    def add_prompt(self, sid: int, tokens: Sequence[int]):
        """Register a sequence by its prompt token ids (automatic prefix
        caching): the longest run of cached full blocks matching the prompt's
        leading blocks is mapped into its table as is (their K/V are already in
        the pools), the remaining tokens get fresh slots.  Returns
        (n_cached, slots): the number of reused tokens and the int64 slots of
        the others, where the caller's ``kv_append`` writes their K/V."""
        st, n_cached, slots = self.alloc.seq_add_with_prompt(sid, tokens)
        self._ok(st)
        return n_cached, np.asarray(slots, dtype=np.int64)

    def cache_stats(self) -> dict:
        """Prefix-cache counters (lookups, hits, cached / evictable blocks, evictions)."""
        return self.alloc.cache_stats()

    def fork(self, parent: int, child: int):
        self._ok(self.alloc.seq_fork(parent, child))

    def free(self, sid: int):
        self._ok(self.alloc.seq_free(sid))

    def table(self, sid: int):
        st, bt, n = self.alloc.seq_block_table(sid)
        self._ok(st)
        return bt, n

    @staticmethod
    def _ok(st):
        if st != B.OK:
            raise B.PagedKVError(st, B.lib.pkv_last_error().decode())

    def plan(self, attend: Sequence[int], write: Optional[Sequence[int]] = None) -> StepPlan:
        """Reserve one new slot for every sequence in ``write`` (default: ``attend``),
        collect copy-on-write pairs, and snapshot the tables of ``attend``."""
        write = list(attend if write is None else write)
        self._check_fits(attend, write)
        st, slots, pairs = self.alloc.seq_append_slots_batch(write)
        self._ok(st)
        st, bt, lens = self.alloc.seq_block_tables_batch(list(attend), self.max_blocks)
        self._ok(st)
        plan = StepPlan(list(attend), slots, pairs.reshape(-1, 2), lens, bt)
        if self.share_prefixes and len(attend) >= self.min_group_size:
            gf, gs = B.find_shared_prefix_groups(bt, lens, self.block_size, self.min_group_size)
            if (gs > 0).any():
                plan.group_first, plan.group_shared = gf, gs
                plan.max_group_size = int(np.diff(gf).max())
                plan.max_shared_len = int(gs.max())
        return plan

    def _check_fits(self, attend: Sequence[int], write) -> None:
        """Fail before any slot is reserved (the step's reservations cannot be
        undone): every sequence of ``attend`` must exist and still fit in
        max_blocks_per_seq blocks after this step's tokens."""
        a = np.asarray(attend, dtype=np.int64)
        st, lens = self.alloc.seq_lens_batch(a)
        self._ok(st)
        if not len(lens):
            return
        ids, counts = np.unique(np.asarray(write, dtype=np.int64), return_counts=True)
        grow = np.zeros(len(a), dtype=np.int64)     # new tokens of each attending sequence
        if len(ids):
            pos = np.minimum(np.searchsorted(ids, a), len(ids) - 1)
            grow = np.where(ids[pos] == a, counts[pos], 0)
        tokens = lens + grow
        blocks = -(-tokens // self.block_size)
        if blocks.max() > self.max_blocks:
            i = int(blocks.argmax())
            raise B.PagedKVError(B.INVALID, "sequence %d would need %d blocks, more than max_blocks_per_seq = %d"
                                 % (int(attend[i]), int(blocks[i]), self.max_blocks))

    def plan_chunk(self, seq_ids: Sequence[int], n_new: Sequence[int]) -> ChunkPlan:
        """Reserve slots for n_new[i] new tokens of seq_ids[i] (a causal chunk:
        draft tokens to verify, or part of a prompt)."""
        ids = np.repeat(np.asarray(seq_ids, dtype=np.int64), np.asarray(n_new, dtype=np.int64))
        self._check_fits(seq_ids, ids)
        st, slots, pairs = self.alloc.seq_append_slots_batch(ids)
        self._ok(st)
        st, bt, lens = self.alloc.seq_block_tables_batch(list(seq_ids), self.max_blocks)
        self._ok(st)
        qs = np.concatenate([[0], np.cumsum(n_new)]).astype(np.int32)
        return ChunkPlan(list(seq_ids), slots, pairs.reshape(-1, 2), lens, bt, qs, int(max(n_new)))

    def launch_chunk(self, d: dict, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, out: torch.Tensor,
                     stream=None):
        """block_copy -> kv_append (all new tokens) -> causal chunk attention."""
        if d["n_cow"]:
            B.block_copy(self.k_pool, self.v_pool, d["cow_pairs"], stream=stream)
        B.kv_append(k_new, v_new, self.k_pool, self.v_pool, d["slot_mapping"], stream=stream)
        B.paged_attention_chunk(out, q, self.k_pool, self.v_pool, d["block_tables"], d["lens"], d["query_start"],
                                d["max_query_len"], partition_size=self.partition_size, workspace=self.workspace,
                                stream=stream)
        return out

    def chunk_to_device(self, p: ChunkPlan) -> dict:
        """Copy a chunk plan to the device (one packed asynchronous copy)."""
        sm, cow, lens, bt, qs = self._pack_h2d([p.slot_mapping, p.cow_pairs, p.lens, p.block_tables, p.query_start])
        return dict(slot_mapping=sm, n_cow=len(p.cow_pairs), cow_pairs=cow if len(p.cow_pairs) else None, lens=lens,
                    block_tables=bt, query_start=qs, max_query_len=p.max_query_len)

    def reserve_chunk_workspace(self, num_tokens: int):
        """Grow the workspace for chunk calls of up to num_tokens query rows."""
        need = B.attention_chunk_workspace_bytes(num_tokens, self.num_q_heads, self.head_dim,
                                                 self.max_blocks * self.block_size, self.partition_size)
        if need > self.workspace.numel():
            self.workspace = torch.empty(need, dtype=torch.uint8, device=self.device)

    def to_device(self, p: StepPlan, non_blocking: bool = False) -> DevicePlan:
        dev = self.device

        def up(a):
            return torch.from_numpy(np.ascontiguousarray(a)).to(dev, non_blocking=non_blocking)
        d = DevicePlan(up(p.slot_mapping), up(p.cow_pairs) if len(p.cow_pairs) else
                       torch.zeros((0, 2), dtype=torch.int32, device=dev),
                       up(p.lens), up(p.block_tables), len(p.cow_pairs))
        if p.has_groups:
            d.group_first, d.group_shared = up(p.group_first), up(p.group_shared)
            d.max_group_size, d.max_shared_len = p.max_group_size, p.max_shared_len
        return d

    # ---------------------------------------------------------- device side
    def launch(self, d: DevicePlan, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
               out: torch.Tensor, stream=None):
        """block_copy (if any pair) -> kv_append -> paged_attention_decode."""
        if d.n_cow:
            B.block_copy(self.k_pool, self.v_pool, d.cow_pairs, stream=stream)
        if self.fp8:
            B.kv_append_fp8(k_new, v_new, self.k_pool, self.v_pool, d.slot_mapping, *self.kv_scales, stream=stream)
        else:
            B.kv_append(k_new, v_new, self.k_pool, self.v_pool, d.slot_mapping, stream=stream)
        return self.attend(d, q, out, stream=stream)

    def attend(self, d: DevicePlan, q: torch.Tensor, out: torch.Tensor, stream=None):
        """The step's attention: the shared-prefix call when the plan found groups."""
        if self.fp8:
            B.paged_attention_decode_fp8(out, q, self.k_pool, self.v_pool, d.block_tables, d.lens, *self.kv_scales,
                                         partition_size=self.partition_size, workspace=self.workspace,
                                         stream=stream)
        elif d.group_shared is not None:
            B.paged_attention_decode_shared(out, q, self.k_pool, self.v_pool, d.block_tables, d.lens,
                                            d.group_first, d.group_shared, d.max_group_size, d.max_shared_len,
                                            partition_size=self.partition_size, workspace=self.workspace,
                                            stream=stream)
        else:
            B.paged_attention_decode(out, q, self.k_pool, self.v_pool, d.block_tables, d.lens,
                                     partition_size=self.partition_size, workspace=self.workspace, stream=stream)
        return out

    def _pin(self, name, like: torch.Tensor):
        t = self._pinned.get(name)
        if t is None or t.shape != like.shape or t.dtype != like.dtype:
            t = torch.empty(like.shape, dtype=like.dtype, pin_memory=True)
            self._pinned[name] = t
        return t

    def step(self, q_host: torch.Tensor, k_new_host: torch.Tensor, v_new_host: torch.Tensor,
             attend: Sequence[int], out_host: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """A full step from host buffers: plan, copy inputs in, run, copy the output back, wait."""
        p = self.plan(attend)
        s = torch.cuda.current_stream() if stream is None else stream
        done = torch.cuda.Event()
        out_host = self.launch_step(p, q_host, k_new_host, v_new_host, out_host, stream=s, out_ready=done)
        done.synchronize()
        return out_host

    # ------------------------------------------------- host-buffer steps
    # A serving loop hands each step's inputs over in host memory and wants
    # the output back in host memory.  launch_step does that for a planned
    # step with one C call (pkv_step_from_host): the plan's arrays, packed into
    # a pinned staging buffer, go in one copy and q / new K / new V in one more
    # (three when they are not laid out in one host buffer like the device
    # block), then block_copy -> kv_append -> attention run and the output
    # comes back in one copy.  The device buffers are made once per layout of
    # the plan's arrays (and per input shape) and the step description is
    # built and checked against their sizes then; a step only refills the
    # staging buffer, sets the host pointers and makes the call.
    #
    # Reuse rules: the device buffers of a layout are reused by later steps of
    # the same layout, so all host-buffer steps of a session go on one stream
    # (stream order then keeps a step's kernels ahead of the next step's
    # copies into the same buffers).  Two staging buffers alternate per
    # layout, and one is refilled only after the step that last used it has
    # completed.

    _MAX_LAYOUTS = 32

    def _layout(self, arrays) -> dict:
        """The next staging set for this layout of plan arrays (made once)."""
        key = tuple((a.dtype.str, a.shape) for a in arrays)
        lay = self._layouts.get(key)
        if lay is None:
            if len(self._layouts) >= self._MAX_LAYOUTS:
                self._layouts.pop(next(iter(self._layouts)))
            offs, total = [], 0
            for a in arrays:
                offs.append(total)
                total += (a.nbytes + 255) // 256 * 256
            total = max(total, 256)
            if self.overlap_input_copies and self._copy_stream is None:
                self._copy_stream = torch.cuda.Stream(device=self.device)
            if self.overlap_output_copies and self._out_stream is None:
                self._out_stream = torch.cuda.Stream(device=self.device)
            sets = []
            for _ in range(2):
                host = torch.empty(total, dtype=torch.uint8, pin_memory=True)
                dev = torch.empty(total, dtype=torch.uint8, device=self.device)
                hv = host.numpy()
                st = {"host": host, "dev": dev, "bytes": total,
                      "hviews": [hv[o:o + a.nbytes].view(a.dtype).reshape(a.shape) for a, o in zip(arrays, offs)],
                      "ptrs": [dev.data_ptr() + o for o in offs], "event": None, "steps": {}, "io": {}}
                if self._copy_stream is not None:
                    # events of the overlapped input copies (recorded once so
                    # that they exist): the set's device buffers are free /
                    # filled
                    st["free"], st["ready"] = torch.cuda.Event(), torch.cuda.Event()
                    st["free"].record(self._copy_stream)
                    st["ready"].record(self._copy_stream)
                if self._out_stream is not None:
                    # the set's output copies are done (its device output
                    # buffers may be written again)
                    st["odone"] = torch.cuda.Event()
                    st["odone"].record(self._out_stream)
                sets.append(st)
            lay = self._layouts[key] = [0, sets]
        lay[0] ^= 1
        return lay[1][lay[0]]

    def _io_buffers(self, st: dict, q_host, k_new_host, v_new_host):
        """Device q / new K / new V / out of a staging set for these host
        shapes (made once per set and shape: the two sets of a layout never
        share them, so one set's input copies can land while the other set's
        step still reads its own)."""
        key = (tuple(q_host.shape), tuple(k_new_host.shape), q_host.dtype, k_new_host.dtype)
        io = st["io"].get(key)
        if io is None:
            if q_host.dim() != 3 or tuple(q_host.shape[1:]) != (self.num_q_heads, self.head_dim):
                raise ValueError("q must be [rows, num_q_heads, head_dim]")
            if k_new_host.dim() != 3 or tuple(k_new_host.shape[1:]) != (self.num_kv_heads, self.head_dim):
                raise ValueError("new K/V must be [T, num_kv_heads, head_dim]")
            if self.fp8:
                if q_host.dtype not in (torch.bfloat16, torch.float16) or k_new_host.dtype != q_host.dtype:
                    raise TypeError("with FP8 pools q and new K/V must be bf16 or f16, of one type")
            elif q_host.dtype != self.k_pool.dtype or k_new_host.dtype != self.k_pool.dtype:
                raise TypeError("q and new K/V must have the pools' element type")
            if len(st["io"]) >= self._MAX_LAYOUTS:
                st["io"].pop(next(iter(st["io"])))
            # q, new K, new V in one device block, each at a 256-byte aligned
            # offset: host inputs laid out the same way go in one copy.
            qb = q_host.numel() * q_host.element_size()
            kb = k_new_host.numel() * k_new_host.element_size()
            ok = (qb + 255) // 256 * 256
            ov = ok + (kb + 255) // 256 * 256
            block = torch.empty(ov + kb, dtype=torch.uint8, device=self.device)
            q = block[:qb].view(q_host.dtype).view(q_host.shape)
            kn = block[ok:ok + kb].view(k_new_host.dtype).view(k_new_host.shape)
            vn = block[ov:ov + kb].view(k_new_host.dtype).view(k_new_host.shape)
            out = torch.empty_like(q)
            io = st["io"][key] = (key, q, kn, vn, out, (block, ok, ov))
        if v_new_host.shape != k_new_host.shape or v_new_host.dtype != k_new_host.dtype:
            raise ValueError("k_new and v_new must have the same shape and element type")
        if not (q_host.is_contiguous() and k_new_host.is_contiguous() and v_new_host.is_contiguous()):
            raise ValueError("host inputs must be contiguous")
        if q_host.is_cuda or k_new_host.is_cuda or v_new_host.is_cuda:
            raise TypeError("launch_step takes host tensors")
        return io

    def _step_struct(self, st: dict, p, io, n_cow: int) -> B.PkvStep:
        """The pkv_step of one staging set and one input shape (host pointers
        left to fill per step)."""
        _, q, kn, vn, out, _ = io
        chunk = isinstance(p, ChunkPlan)
        ins = (B.PkvCopy * 4)()
        ins[0] = B.PkvCopy(st["dev"].data_ptr(), st["host"].data_ptr(), st["bytes"])
        for c, t in zip(ins[1:], (q, kn, vn)):
            c.dst, c.bytes = t.data_ptr(), t.numel() * t.element_size()
        outs = (B.PkvCopy * 1)()
        outs[0].src, outs[0].bytes = out.data_ptr(), out.numel() * out.element_size()
        ptrs = st["ptrs"]
        rest = ptrs[3 + (1 if n_cow else 0):]
        kind = B.STEP_CHUNK if chunk else B.STEP_DECODE_FP8 if self.fp8 else \
            B.STEP_DECODE_SHARED if p.has_groups else B.STEP_DECODE
        k_scale, v_scale = self.kv_scales if self.fp8 else (1.0, 1.0)
        step = B.PkvStep(
            struct_size=ctypes.sizeof(B.PkvStep), kind=kind, in_=ins, n_in=4, out=outs, n_out=1,
            k_pool=self.k_pool.data_ptr(), v_pool=self.v_pool.data_ptr(), num_blocks=self.num_blocks,
            num_kv_heads=self.num_kv_heads, head_dim=self.head_dim, block_size=self.block_size,
            dtype=B._dt(q), k_scale=float(k_scale), v_scale=float(v_scale),
            pairs=ptrs[3] if n_cow else None, num_pairs=n_cow,
            k_new=kn.data_ptr(), v_new=vn.data_ptr(), slot_mapping=ptrs[0], num_tokens=len(p.slot_mapping),
            attn_out=out.data_ptr(), q=q.data_ptr(), block_tables=ptrs[2],
            max_blocks_per_seq=p.block_tables.shape[1], context_lens=ptrs[1], num_seqs=len(p.lens),
            num_q_heads=self.num_q_heads, scale=0.0, partition_size=self.partition_size,
            workspace=self.workspace.data_ptr(), workspace_bytes=self.workspace.numel(),
            group_first=rest[0] if (not chunk and p.has_groups) else None,
            group_shared=rest[1] if (not chunk and p.has_groups) else None,
            num_groups=len(p.group_shared) if (not chunk and p.has_groups) else 0,
            max_group_size=int(p.max_group_size) if not chunk else 0,
            max_shared_len=int(p.max_shared_len) if not chunk else 0,
            query_start=rest[0] if chunk else None, max_query_len=int(p.max_query_len) if chunk else 0)
        if self._copy_stream is not None:   # input copies on the session's copy stream
            step.copy_stream = self._copy_stream.cuda_stream
            step.inputs_free, step.inputs_ready = st["free"].cuda_event, st["ready"].cuda_event
        if self._out_stream is not None:    # output copies on the session's output stream
            step.out_stream, step.outputs_done = self._out_stream.cuda_stream, st["odone"].cuda_event
        step._copies = (ins, outs)          # the arrays the struct points to stay alive with it
        return step

    def launch_step(self, p, q_host: torch.Tensor, k_new_host: torch.Tensor, v_new_host: torch.Tensor,
                    out_host: Optional[torch.Tensor] = None, stream=None, out_ready=None) -> torch.Tensor:
        """Issue one planned step (a StepPlan, or a ChunkPlan) from host
        buffers without waiting: the plan and the inputs go to the device,
        block_copy -> kv_append -> attention run, and the output is copied into
        ``out_host`` (pinned; if None, the session's own buffer, which the next
        call without one reuses: with several steps in flight, pass one buffer
        per step) -- complete once ``stream`` reaches this point.  q_host
        [rows, num_q_heads, head_dim]; k/v_new_host [tokens written,
        num_kv_heads, head_dim]; pinned host memory lets the copies run
        asynchronously.  Inputs that sit in one host buffer -- q, then new K
        at the next 256-byte boundary after q, then new V at the next after new
        K -- are sent with a single copy.  With ``overlap_input_copies`` the
        input copies run on the session's copy stream, and ``stream``'s
        kernels wait for them; the host buffers must stay untouched until
        ``stream`` reaches the end of the step either way.  ``out_ready`` (a
        torch.cuda.Event, optional) is recorded where the output copy is
        complete: on ``stream``, or with ``overlap_output_copies`` on the
        session's output stream -- then ``stream`` reaching the end of the
        step does not mean the output has arrived, and out_ready is how to
        wait for it."""
        s = torch.cuda.current_stream() if stream is None else stream
        chunk = isinstance(p, ChunkPlan)
        T = len(p.slot_mapping)
        rows = T if chunk else len(p.seq_ids)
        if q_host.shape[0] != rows or k_new_host.shape[0] != T:
            raise ValueError("q needs one row per %s and new K/V one per written token"
                             % ("new token" if chunk else "attending sequence"))
        n_cow = len(p.cow_pairs)
        arrays = [p.slot_mapping, p.lens, p.block_tables] + ([p.cow_pairs] if n_cow else [])
        if chunk:
            arrays.append(p.query_start)
        elif p.has_groups:
            arrays += [p.group_first, p.group_shared]
        st = self._layout(arrays)
        io = self._io_buffers(st, q_host, k_new_host, v_new_host)
        out = io[4]
        if out_host is None:
            out_host = self._pin("out", out)
        elif out_host.shape != out.shape or out_host.dtype != out.dtype or out_host.is_cuda or \
                not out_host.is_contiguous():
            raise ValueError("out_host must be a contiguous host tensor of q's shape and element type")
        if st["event"] is not None:
            st["event"].synchronize()           # the step that last used this staging set is done
        for hv, a in zip(st["hviews"], arrays):
            np.copyto(hv, a, casting="no")
        step = st["steps"].get(io[0])
        if step is None:
            step = st["steps"][io[0]] = self._step_struct(st, p, io, n_cow)
        ins, outs = step._copies
        block, ok, ov = io[5]
        qp, kp, vp = q_host.data_ptr(), k_new_host.data_ptr(), v_new_host.data_ptr()
        if kp - qp == ok and vp - qp == ov:      # inputs packed like the device block: one copy
            ins[1].src, ins[1].bytes = qp, block.numel()
            step.n_in = 2
        else:
            ins[1].src, ins[1].bytes = qp, q_host.numel() * q_host.element_size()
            ins[2].src, ins[3].src = kp, vp
            step.n_in = 4
        outs[0].dst = out_host.data_ptr()
        if chunk:                                # the plan's values that its layout does not fix
            step.max_query_len = int(p.max_query_len)
        elif p.has_groups:
            step.max_group_size, step.max_shared_len = int(p.max_group_size), int(p.max_shared_len)
        B.raw_call("pkv_step_from_host", ctypes.byref(step), s.cuda_stream)
        if st["event"] is None:
            st["event"] = torch.cuda.Event()
        st["event"].record(s)
        if out_ready is not None:
            out_ready.record(self._out_stream if self._out_stream is not None else s)
        return out_host


    def upload(self, p: StepPlan) -> DevicePlan:
        """Copy a plan to the device: its arrays packed into one pinned staging
        buffer and sent with a single asynchronous copy."""
        arrs = [p.slot_mapping, p.cow_pairs, p.lens, p.block_tables]
        if p.has_groups:
            arrs += [p.group_first, p.group_shared]
        dv = self._pack_h2d(arrs)
        d = DevicePlan(dv[0], dv[1], dv[2], dv[3], len(p.cow_pairs))
        if p.has_groups:
            d.group_first, d.group_shared = dv[4], dv[5]
            d.max_group_size, d.max_shared_len = p.max_group_size, p.max_shared_len
        return d

    def _pack_h2d(self, arrays) -> list:
        """One host->device copy for several host arrays (each at a 256-byte
        aligned offset); returns device views of the original shapes/dtypes.
        Two staging buffers alternate, and a buffer is refilled only after its
        previous copy has completed, so calls need no synchronisation."""
        arrays = [np.ascontiguousarray(a) for a in arrays]
        offs, total = [], 0
        for a in arrays:
            offs.append(total)
            total += (a.nbytes + 255) // 256 * 256
        total = max(total, 256)
        k = self._stage_next = getattr(self, "_stage_next", 0) ^ 1
        stage, ev = self._pinned.get(("stage", k), (None, None))
        if ev is not None:
            ev.synchronize()
        if stage is None or stage.numel() < total:
            stage = torch.empty(max(total, 1 << 16), dtype=torch.uint8, pin_memory=True)
        sv = stage.numpy()
        for a, o in zip(arrays, offs):
            sv[o:o + a.nbytes] = a.reshape(-1).view(np.uint8)
        dev = stage[:total].to(self.device, non_blocking=True)
        ev = torch.cuda.Event()
        ev.record()
        self._pinned[("stage", k)] = (stage, ev)
        return [dev[o:o + a.nbytes].view(torch.from_numpy(a[:0].reshape(-1)).dtype).view(a.shape)
                for a, o in zip(arrays, offs)]
