#!/usr/bin/env python
"""Paged KV cache decode benchmark (one JSON line on rank 0).

A step is one decode step of one layer for a whole batch: every sequence gets
the slot of its next token from the block allocator (copy-on-write pairs
where a shared, partly filled block is written), the copies are made
(block_copy), the new K/V are written (kv_append) and every query attends to
its cached tokens through its block table (paged_attention_decode).  Lengths
grow by one token per step.

value  -- algorithmic bytes of the step (unique K/V bytes the attention must
          read, shared blocks counted once, plus q, out, tables, split-K
          workspace, appended and copied bytes) / device time, inputs already
          resident in HBM (the step's plan is made on the host beforehand).
e2e    -- the same metric through DecodeSession.launch_step: allocator on the
          host, every step's inputs copied in from pinned host memory and its
          output copied back to pinned host memory and waited for, two steps
          in flight (--e2e-in-flight; the line also carries the figure with
          the host waiting for each output before the next step goes); input
          and output copies on streams of the session's own, overlapping
          the neighbouring steps' kernels (--e2e-serial-output keeps the
          output copy on the kernels' stream).

The headline workload (``--config``, default ``llama3_gqa_bs16``: 128
sequences x 8192 tokens, 32 query / 8 kv heads, the largest one-GPU decode
workload) gives the line's value, roofline, e2e and CPU baseline; the
``targets`` object carries the same device and end-to-end numbers for the
workloads timed after it in the same run (by default the shared-system-prompt
and 100k-token-context workloads, which carry the >= 70 % of HBM peak target,
and the Llama-2-7B-shaped MHA layer).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
       [--targets A,B|none] [--impl ours|reference].  Under torchrun each
rank runs its own replica (own pool, own sequences; no collective on the data
path): weak scaling.  ``--impl reference`` times the CPU oracle instead (rank
0 only) and names the same workload in its ``config``.
"""
import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "paged decode attention HBM GB/s (% of B200 peak) and seq-steps/s per layer"
# Headline workload: the largest one-GPU decode configuration (Llama-3-8B-shaped
# grouped-query decode, 128 sequences x 8192 tokens, 4.29 GB of K/V per call).
DEFAULT_CONFIG = "llama3_gqa_bs16"
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------- accounting
def chunk_ws_bytes(lens, query_start, Hq: int, D: int, P: int) -> int:
    """Split-K partials written and read back by a causal chunk call."""
    total = 0
    for s in range(len(lens)):
        L, n = int(lens[s]), int(query_start[s + 1] - query_start[s])
        if -(-L // P) <= 1:
            continue
        pos = L - n + np.arange(n)
        total += int((pos // P + 1).sum()) * Hq * (D + 2) * 4 * 2
    return total


def attention_bytes(bt: np.ndarray, lens: np.ndarray, Hq: int, Hkv: int, D: int, bs: int, elt: int,
                    P: int, shared=None, q_rows=None, q_elt=None) -> dict:
    """Algorithmic bytes of one decode-attention call.

    K/V: every physical (block, kv head) tile covered by some context counts
    once, with the number of tokens covered (a shared prefix is read once by
    the algorithm's definition of "unique"); plus q and out, the block-table
    entries and context lengths read, and the split-K partials written and
    read back.
    """
    S = len(lens)
    lens = np.asarray(lens, dtype=np.int64)
    nb = -(-lens // bs)
    j = np.arange(bt.shape[1])[None, :]
    used = j < nb[:, None]
    cov = np.clip(lens[:, None] - j * bs, 0, bs)[used]       # tokens covered in each used entry
    blk = bt[used].astype(np.int64)
    best = np.zeros(int(blk.max()) + 1 if blk.size else 1, dtype=np.int64)
    np.maximum.at(best, blk, cov)                            # a block shared by several contexts counts once
    tok = int(best.sum())
    kv = 2 * Hkv * D * elt * tok
    logical = 2 * Hkv * D * elt * int(lens.sum())
    qo = 2 * (S if q_rows is None else q_rows) * Hq * D * (elt if q_elt is None else q_elt)
    tables = 4 * int(nb.sum()) + 4 * S
    sh = np.zeros(S, dtype=np.int64) if shared is None else np.asarray(shared, dtype=np.int64)
    nparts = -(-sh // P) + -(-(lens - sh) // P)
    merged = (nparts > 1) | (sh > 0)
    ws = int((2 * nparts * Hq * (D + 2) * 4)[merged].sum())
    # KV memory utilisation: tokens held / slots of the physical blocks in use
    util = tok / max(1, int((best > 0).sum()) * bs)
    return dict(kv=kv, logical_kv=logical, total=kv + qo + tables + ws, ws=ws, kv_util=util)


def append_bytes(T, Hkv, D, elt):
    return 2 * 2 * T * Hkv * D * elt + 8 * T


def copy_bytes(n_pairs, Hkv, bs, D, elt):
    return 2 * 2 * n_pairs * Hkv * bs * D * elt


# ------------------------------------------------------------------- workload
class Workload:
    """A batch laid out in the pool plus the session that drives its steps."""

    def __init__(self, shape, seed, device, partition_size, overlap_output_copies=True):
        import paged_kv_cache_405_b200 as pkv
        self.shape = shape
        self.batch = synth.make_batch(shape, device=device, seed=seed)
        b = self.batch
        self.P = partition_size or shape.partition_size
        self.session = pkv.DecodeSession(b.k_pool, b.v_pool, shape.Hq, b.max_blocks, free_order=b.free_order,
                                         partition_size=self.P, max_batch=shape.S,
                                         overlap_output_copies=overlap_output_copies,
                                         kv_scales=(shape.kv_scale, shape.kv_scale) if shape.kv_fp8 else None)
        ss = self.session
        if shape.prefix:
            ss.add(-1, shape.prefix)                       # the prompt, stored once
            prefix, _ = ss.table(-1)
        for s in range(shape.S):
            if shape.prefix:
                ss.add(s, int(b.lens[s]) - shape.prefix, shared_prefix=prefix, prefix_tokens=shape.prefix)
            else:
                ss.add(s, int(b.lens[s]))
            t, _ = ss.table(s)
            exp = b.block_tables[s][b.block_tables[s] >= 0].tolist()
            if t != exp:
                raise RuntimeError("allocator disagrees with the batch layout for seq %d" % s)
        if shape.prefix:
            ss.free(-1)
        self.parents = list(range(shape.S))
        if shape.chunk:
            ss.reserve_chunk_workspace(shape.S * shape.chunk)
        self.elt = b.k_pool.element_size()     # pool element (1 byte for FP8 codes)
        self.q_elt = b.q.element_size()
        self.eff_P = pkv.attention_partition_size(shape.S, shape.Hq, shape.Hkv, shape.D,
                                                  b.max_blocks * shape.bs, self.P)
        self.next_child = shape.S

    def plan(self):
        """Host work of one step: a StepPlan, or a ChunkPlan for chunk workloads."""
        sh, ss = self.shape, self.session
        if sh.chunk:
            return ss.plan_chunk(self.parents, [sh.chunk] * len(self.parents))
        children = []
        if sh.beams:
            for p in self.parents:
                for _ in range(sh.beams - 1):
                    ss.fork(p, self.next_child)
                    children.append(self.next_child)
                    self.next_child += 1
        # children write first (each copies the shared last block); the parent
        # is then the block's only user and writes in place.
        if sh.beams:
            write = []
            for i, p in enumerate(self.parents):
                write += children[i * (sh.beams - 1):(i + 1) * (sh.beams - 1)]
                write.append(p)
        else:
            write = self.parents
        plan = ss.plan(self.parents, write)
        for c in children:
            ss.free(c)
        return plan

    def to_device(self, plan):
        return self.session.chunk_to_device(plan) if self.shape.chunk else self.session.to_device(plan)

    def upload(self, plan):
        return self.session.chunk_to_device(plan) if self.shape.chunk else self.session.upload(plan)

    def launch(self, d, q, kn, vn, out):
        if self.shape.chunk:
            return self.session.launch_chunk(d, q, kn, vn, out)
        return self.session.launch(d, q, kn, vn, out)

    def step_bytes(self, plan):
        sh = self.shape
        if sh.chunk:
            a = attention_bytes(plan.block_tables, plan.lens, sh.Hq, sh.Hkv, sh.D, sh.bs, self.elt, self.eff_P,
                                q_rows=len(plan.slot_mapping))
            a["ws"] = chunk_ws_bytes(plan.lens, plan.query_start, sh.Hq, sh.D, self.eff_P)
            a["total"] = a["kv"] + 2 * len(plan.slot_mapping) * sh.Hq * sh.D * self.elt + a["ws"] + \
                4 * int(sum(-(-int(L) // sh.bs) for L in plan.lens)) + 8 * len(plan.lens)
            total = a["total"] + append_bytes(len(plan.slot_mapping), sh.Hkv, sh.D, self.elt) + \
                copy_bytes(len(plan.cow_pairs), sh.Hkv, sh.bs, sh.D, self.elt)
            return total, a
        shared = None
        if plan.has_groups:   # per-sequence shared length of its group
            shared = np.repeat(plan.group_shared, np.diff(plan.group_first))
        a = attention_bytes(plan.block_tables, plan.lens, sh.Hq, sh.Hkv, sh.D, sh.bs, self.elt, self.eff_P,
                            shared=shared, q_elt=self.q_elt)
        # append: new K/V read in the q/out type, written as pool elements
        total = a["total"] + append_bytes(len(plan.slot_mapping), sh.Hkv, sh.D, self.elt) // 2 + \
            append_bytes(len(plan.slot_mapping), sh.Hkv, sh.D, self.q_elt) // 2 + \
            copy_bytes(len(plan.cow_pairs), sh.Hkv, sh.bs, sh.D, self.elt)
        return total, a


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------- profiles data
def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_405_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh")):
            h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(config):
    """DRAM bytes per decode call from the committed ncu summary, if it was
    taken on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    src = kernel_source_hash()
    for line in open(path):
        f = line.split()
        if len(f) >= 3 and not line.startswith("#") and f[0] == config and f[1] == src:
            return float(f[2])
    return None


NOMINAL_HBM_GBS = 8000.0   # B200 HBM3e nominal, for context beside the measured copy bandwidth


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        return float(json.load(open(path))["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------- CPU oracle leg
def oracle_sample(batch, budget_s, threads):
    """Time the CPU oracle on whole sequences of the batch until ~budget_s of
    work; returns (KV GB/s, seq-steps/s, description)."""
    import oracle
    S, Hq = batch.shape.S, batch.shape.Hq
    q = batch.q.cpu()
    k = batch.k_pool.cpu()
    v = batch.v_pool.cpu()
    elt = k.element_size()
    bytes_done, secs, seqs, passes = 0, 0.0, 0, 0
    order = np.random.default_rng(0).permutation(S)
    while secs < budget_s:
        for s in order:
            L = int(batch.lens[s])
            items = [(int(s), h) for h in range(Hq)]
            t0 = time.perf_counter()
            if batch.shape.kv_fp8:
                oracle.paged_attention_kv(q, k, v, batch.shape.kv_scale, batch.shape.kv_scale, batch.block_tables,
                                          batch.lens, items=items, threads=threads)
            else:
                oracle.paged_attention(q, k, v, batch.block_tables, batch.lens, items=items, threads=threads)
            secs += time.perf_counter() - t0
            bytes_done += 2 * L * batch.shape.D * elt * Hq
            seqs += 1
            if secs >= budget_s:
                break
        passes += 1
    desc = "%d sequence-steps over %d pass(es) of the %d-sequence batch (every query head; %.2f GB of K/V " \
        "reads), fp64 oracle, %d threads" % (seqs, passes, S, bytes_done / 1e9, threads)
    return bytes_done / secs / 1e9, seqs / secs, desc, secs


def cpu_model() -> str:
    """The host CPU's model name (for the CPU-baseline record)."""
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ------------------------------------------------------------------- runners
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def workload_shape(args, name=None):
    shape = synth.CONFIGS[args.config if name is None else name]
    if args.batch:
        shape = synth.shrink(shape, S=args.batch)
    # --prefix overrides the shared-prompt length of the headline workload only
    if getattr(args, "prefix", 0) and shape.prefix and (name is None or name == args.config):
        shape = synth.shrink(shape, prefix=args.prefix)
    # room in every table and in the pool for the tokens the run appends
    grow = (max(args.warmup, 10) + args.steps + 8) * max(1, shape.chunk)
    if grow > shape.reserve_tokens:
        shape = synth.shrink(shape, reserve_tokens=grow)
    return shape


def workload_config(name, shape, batch, args, world) -> dict:
    """The ``config`` object of a bench line: the workload, its shape and how
    L2 is handled.  Both arms build it from the same seeded batch, so the
    reference arm's line names exactly the workload this arm times."""
    pool_gb = 2 * batch.k_pool.numel() * batch.k_pool.element_size() / 1e9
    tag = ("" if not args.batch else "@batch%d" % args.batch) + \
        ("" if not (getattr(args, "prefix", 0) and shape.prefix) else "@prefix%d" % shape.prefix)
    return {"workload": name + tag,
            "description": shape.description, "batch": shape.S,
            "q_heads": shape.Hq, "kv_heads": shape.Hkv, "head_dim": shape.D, "block_size": shape.bs,
            "kv_dtype": "e4m3" if shape.kv_fp8 else shape.dtype,
            "partition_size": args.partition_size or shape.partition_size,
            "mean_context": round(float(np.mean(batch.lens)), 1),
            "new_tokens_per_seq": max(1, shape.chunk),
            "l2": "inputs larger than L2 (K/V pool %.2f GB per rank)" % pool_gb,
            "parallelism": "replica per GPU" if world > 1 else "1 GPU"}


def measure_workload(name, args, world, rank, local, e2e=True):
    """Time K decode steps of workload ``name`` after W warm-up steps, inputs
    resident in HBM (CUDA events on the launching stream, max over ranks),
    then the same steps end to end from host buffers.  Returns the numbers
    of one bench line (without the CPU baseline)."""
    import paged_kv_cache_405_b200 as pkv
    shape = workload_shape(args, name)
    dev = torch.device("cuda", local)
    wl = Workload(shape, shape.seed + rank, dev, args.partition_size)
    ss = wl.session
    K, W = args.steps, args.warmup
    dt = synth.DTYPES[shape.dtype]
    config = workload_config(name, shape, wl.batch, args, world)

    # ---- plan every step on the host first (device-resident inputs)
    plans, step_bytes, attn_bytes = [], [], []
    for i in range(W + K):
        p = wl.plan()
        plans.append(wl.to_device(p))
        tb, a = wl.step_bytes(p)
        step_bytes.append(tb)
        attn_bytes.append(a)
    T = len(plans[0]["slot_mapping"] if shape.chunk else plans[0].slot_mapping)
    Tq = shape.S * max(1, shape.chunk)
    inputs = []
    for i in range(W + K):
        q = synth.randn((Tq, shape.Hq, shape.D), torch.Generator(device=dev).manual_seed(7907 * i + rank), dt, dev)
        kn = synth.randn((T, shape.Hkv, shape.D), torch.Generator(device=dev).manual_seed(7919 * i + rank), dt, dev)
        vn = synth.randn((T, shape.Hkv, shape.D), torch.Generator(device=dev).manual_seed(7919 * i + rank + 1),
                         dt, dev)
        inputs.append((q, kn, vn))
    out = torch.empty_like(inputs[0][0])
    stream = torch.cuda.current_stream()

    if args.nvtx:
        pkv.set_nvtx(True)      # one range per library call, inside one per step

    def run_step(i, ev=None):
        if not args.nvtx:
            return step_calls(i, ev)
        torch.cuda.nvtx.range_push("decode_step")
        try:
            return step_calls(i, ev)
        finally:
            torch.cuda.nvtx.range_pop()

    def step_calls(i, ev=None):
        d = plans[i]
        q, kn, vn = inputs[i]
        if shape.chunk:
            if d["n_cow"]:
                pkv.block_copy(ss.k_pool, ss.v_pool, d["cow_pairs"])
            pkv.kv_append(kn, vn, ss.k_pool, ss.v_pool, d["slot_mapping"])
            if ev is not None:
                ev[0].record(stream)
            pkv.paged_attention_chunk(out, q, ss.k_pool, ss.v_pool, d["block_tables"], d["lens"],
                                      d["query_start"], d["max_query_len"], partition_size=wl.P,
                                      workspace=ss.workspace)
        else:
            if d.n_cow:
                pkv.block_copy(ss.k_pool, ss.v_pool, d.cow_pairs)
            if ss.fp8:
                pkv.kv_append_fp8(kn, vn, ss.k_pool, ss.v_pool, d.slot_mapping, *ss.kv_scales)
            else:
                pkv.kv_append(kn, vn, ss.k_pool, ss.v_pool, d.slot_mapping)
            if ev is not None:
                ev[0].record(stream)
            ss.attend(d, q, out)
        if ev is not None:
            ev[1].record(stream)

    for i in range(W):
        run_step(i)
    torch.cuda.synchronize()
    if pkv.device_error() != 0:
        raise RuntimeError("device-side check failed during warm-up (%s)" % name)
    attn_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    # Clocks are sampled while the GPU is busy: repeat the last warm-up step
    # (its writes are idempotent) for ~0.5 s right before the timed region.
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run_step(W - 1)
    e1.record(stream)
    torch.cuda.synchronize()
    n_busy = int(min(20000, max(1, args.clock_warm_s * 1e3 / max(e0.elapsed_time(e1), 1e-3))))
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.15)
    for _ in range(n_busy):
        run_step(W - 1)
    launches0 = pkv.launch_count()
    t0.record(stream)
    for j in range(K):
        run_step(W + j, attn_ev[j])
    t1.record(stream)
    torch.cuda.synchronize()
    launches = pkv.launch_count() - launches0
    clk = clocks.stop()
    barrier(world)
    if pkv.device_error() != 0:
        raise RuntimeError("device-side check failed during the timed steps (%s)" % name)
    ms = t0.elapsed_time(t1)
    attn_ms = [a.elapsed_time(b) for a, b in attn_ev]
    ms_max = max_over_ranks(ms, world)
    timed_bytes = float(sum(step_bytes[W:]))
    total_bytes = sum_over_ranks(timed_bytes, world)
    value = total_bytes / (ms_max * 1e-3) / 1e9
    seq_steps = sum_over_ranks(float(shape.S * K), world) / (ms_max * 1e-3)

    # ---- roofline of the decode-attention call (attention kernel + its split-K merge or reduce)
    peak, peak_kind = measured_hbm_peak()
    a_bytes = float(np.mean([a["total"] for a in attn_bytes[W:]]))
    a_s = max_over_ranks(float(np.mean(attn_ms)), world) * 1e-3
    achieved = a_bytes / a_s / 1e9
    traffic = recorded_traffic(name)
    launch = {"effective_partition_size": wl.eff_P,
              "shared_prefix_groups": int((plans[W].group_shared > 0).sum().item())
              if not shape.chunk and plans[W].group_shared is not None else 0,
              **({"nvtx_ranges": True} if args.nvtx else {})}
    res = {
        "value": round(value, 1), "ms_per_step": round(ms_max / K, 4), "config": config, "launch": launch,
        "dtype": shape.dtype + ("+e4m3-kv" if shape.kv_fp8 else ""),
        "pct_of_peak": round(100 * value / peak, 1),
        "seq_steps_per_s": round(seq_steps, 1),
        "kv_utilisation": round(float(np.mean([a["kv_util"] for a in attn_bytes[W:]])), 4),
        "attention_us": round(a_s * 1e6, 2),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic, "peak_source": peak_kind,
                     "frac_of_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
                     "kernel": "paged_attention_decode (the call's kernels: attention, and the split-K reduce where the "
                               "attention kernel does not merge its own partials)",
                     "algorithmic_bytes": round(a_bytes)},
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    res["e2e"] = None
    if e2e and not args.no_e2e:
        del wl, ss, plans, inputs, out
        torch.cuda.empty_cache()
        depth = max(1, args.e2e_in_flight)
        wl2 = Workload(shape, shape.seed + rank, dev, args.partition_size, not args.e2e_serial_output)
        res["e2e"] = run_e2e(args, wl2, world, rank, dev, depth)
        del wl2
        torch.cuda.empty_cache()
        if depth > 1:           # the same steps with the host waiting before each issue, for comparison
            wl3 = Workload(shape, shape.seed + rank, dev, args.partition_size, not args.e2e_serial_output)
            one = run_e2e(args, wl3, world, rank, dev, 1)
            res["e2e"]["one_in_flight"] = {k: one[k] for k in ("value", "unit", "ms_per_step", "ms_per_step_median")}
            del wl3
    torch.cuda.empty_cache()
    return res


# Configurations timed beside the headline in the default run: the two that
# carry the >= 70 % target (shared system prompt, 100k-token contexts) and
# the Llama-2-7B-shaped MHA layer.
DEFAULT_TARGETS = ("llama13b_prefix", "longctx_beam", "llama7b")


def target_names(args):
    if args.targets == "none":
        return []
    if args.targets:
        return [t for t in args.targets.split(",") if t]
    if args.batch or args.config != DEFAULT_CONFIG:
        return []
    return list(DEFAULT_TARGETS)


def run_ours(args, world, rank, local):
    head = measure_workload(args.config, args, world, rank, local)
    targets = {}
    for name in target_names(args):
        r = measure_workload(name, args, world, rank, local)
        targets[name] = {k: r[k] for k in ("value", "ms_per_step", "attention_us", "seq_steps_per_s",
                                           "pct_of_peak", "roofline", "e2e", "clocks", "config", "dtype")}
    if rank != 0:
        return None
    line = {
        "metric": METRIC, "value": head["value"], "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": head["dtype"],
        "data": "synthetic (seeded N(0,1) K/V/q; pages' workload shapes)",
        "config": head["config"], "launch": head["launch"],
        "pct_of_peak": head["pct_of_peak"], "seq_steps_per_s": head["seq_steps_per_s"],
        "kv_utilisation": head["kv_utilisation"], "attention_us": head["attention_us"],
        "roofline": head["roofline"], "e2e": head["e2e"], "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
    }
    if targets:
        line["targets"] = targets
    if world == 1 and not args.no_cpu_baseline:
        shape = workload_shape(args)
        hb = host_batch(shape, shape.seed + rank)
        v, sps, desc, secs = oracle_sample(hb, args.cpu_seconds, threads=os.cpu_count())
        v1, sps1, _, secs1 = oracle_sample(hb, max(1.0, args.cpu_seconds / 4), threads=1)
        line["cpu_baseline"] = {"value": round(v, 3), "unit": "GB/s", "cores": os.cpu_count(),
                                "kind": "oracle", "sample": desc, "seq_steps_per_s": round(sps, 3),
                                "seconds": round(secs, 1), "cpu_model": cpu_model(),
                                "single_thread": {"value": round(v1, 3), "seq_steps_per_s": round(sps1, 3),
                                                  "seconds": round(secs1, 1)}}
    return line


def host_batch(shape, seed):
    """The same workload generated on the host for the CPU oracle."""
    return synth.make_batch(shape, device="cpu", seed=seed)


def run_e2e(args, wl, world, rank, dev, depth=1):
    """The same steps through the public API from host buffers: every step's
    q / new K / new V arrive in pinned host memory, DecodeSession.launch_step
    sends them and the step's plan to the device, runs block_copy, kv_append
    and attention and copies the output back to pinned host memory, and the
    host waits for every step's output.  ``depth`` steps are in flight: the
    host issues step i, plans step i+1, and then waits for the output of step
    i - depth + 1 (depth 1: the host waits for each step's output before it
    issues the next; depth 2: while it reads one step's output, the next
    step's copies and kernels are already queued, as a serving loop with two
    batches -- or two layers -- in flight would).  The input copies go on the
    session's copy stream, the kernels on the current stream and the output
    copies on the session's output stream (overlap_output_copies), so one
    step's output can cross to the host while the next step's kernels run;
    the host waits for each output through the event launch_step records
    once that copy is complete."""
    import paged_kv_cache_405_b200 as pkv
    shape = wl.shape
    ss = wl.session
    K, W = args.steps, max(args.warmup, 10)      # untimed steps: at least 10 (staging for every layout made)
    dt = synth.DTYPES[shape.dtype]
    T = shape.S * max(1, shape.beams, shape.chunk)
    Tq = shape.S * max(1, shape.chunk)
    shapes = [(Tq, shape.Hq, shape.D), (T, shape.Hkv, shape.D), (T, shape.Hkv, shape.D)]
    esz = torch.empty((), dtype=dt).element_size()
    offs, total = [], 0
    for sh_ in shapes:
        offs.append(total)
        total += (int(np.prod(sh_)) * esz + 255) // 256 * 256
    host_inputs = []        # per step: q, new K, new V in one pinned host buffer
    for i in range(W + K):
        g = torch.Generator().manual_seed(104729 * (i + 1) + rank)
        buf = torch.empty(total, dtype=torch.uint8, pin_memory=True)
        views = []
        for sh_, o in zip(shapes, offs):
            t = synth.randn(sh_, g, dt, "cpu")
            buf[o:o + t.numel() * esz].copy_(t.reshape(-1).view(torch.uint8))
            views.append(buf[o:o + t.numel() * esz].view(dt).view(sh_))
        host_inputs.append((buf, views))
    outs = [torch.empty(shapes[0], dtype=dt, pin_memory=True) for _ in range(depth)]
    out_host = outs[0]
    stream = torch.cuda.current_stream()
    plans = []

    step_ev = []

    def run(first, n, events=False):
        p = wl.plan()
        plans.append(p)
        pending = []            # steps whose output the host has not waited for, oldest first
        for i in range(first, first + n):
            if events:
                step_ev.append(torch.cuda.Event(enable_timing=True))
                step_ev[-1].record(stream)
            done = torch.cuda.Event()
            ss.launch_step(p, *host_inputs[i][1], out_host=outs[i % depth], stream=stream, out_ready=done)
            pending.append(done)
            if i + 1 < first + n:
                p = wl.plan()       # host work of the next step, overlapping this step's kernels
                plans.append(p)
            while len(pending) >= depth:
                pending.pop(0).synchronize()   # that step's output is on the host
        for e in pending:
            e.synchronize()

    def plan_bytes(p):
        arrs = [p.slot_mapping, p.lens, p.block_tables] + ([p.cow_pairs] if len(p.cow_pairs) else [])
        if shape.chunk:
            arrs.append(p.query_start)
        elif p.has_groups:
            arrs += [p.group_first, p.group_shared]
        return max(256, sum((np.asarray(a).nbytes + 255) // 256 * 256 for a in arrs))

    run(0, W)
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    run(W, K, events=True)
    t1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), world)
    per_step = [a.elapsed_time(b) for a, b in zip(step_ev, step_ev[1:] + [t1])]
    timed = plans[W:]
    nbytes = [wl.step_bytes(p)[0] for p in timed]
    tot = sum_over_ranks(float(sum(nbytes)), world)
    if pkv.device_error() != 0:
        raise RuntimeError("device-side check failed during the end-to-end steps")
    h2d = sum(int(np.prod(sh_)) * esz for sh_ in shapes) + plan_bytes(timed[-1])
    d2h = out_host.numel() * out_host.element_size()
    return {"value": round(tot / (ms * 1e-3) / 1e9, 1), "unit": "GB/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": round(ms / K, 4),
            "ms_per_step_median": round(float(np.median(per_step)), 4), "steps_in_flight": depth,
            "api": "DecodeSession.plan (next step planned during this one) + DecodeSession.launch_step (H2D of "
                   "the inputs from pinned host memory and of the plan on a copy stream, block_copy/kv_append/"
                   "attention, D2H of the output on an output stream); the host waits for every step's output, %s" %
                   ("before it issues the next step" if depth == 1 else
                    "with %d steps in flight" % depth)}


def run_reference(args, world, rank):
    """The CPU oracle as the reference arm: each step is a bounded sample of the workload."""
    if rank != 0:
        return None
    shape = workload_shape(args)
    batch = synth.make_batch(shape, device="cpu")
    per = max(0.5, args.reference_step_seconds)
    for _ in range(args.warmup):
        oracle_sample(batch, per / 4, threads=os.cpu_count())
    vals, secs = [], []
    desc = ""
    for _ in range(args.steps):
        v, sps, desc, s = oracle_sample(batch, per, threads=os.cpu_count())
        vals.append(v)
        secs.append(s)
    value = float(np.mean(vals))
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * float(np.mean(secs)), 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same seeded workload, host copy)",
        "config": workload_config(args.config, shape, batch, args, world),
        "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": os.cpu_count(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_allocator_bench(args):
    """Host-only serving simulation of the block allocator with automatic
    prefix caching: requests whose prompts start with one of a few system
    prompts (512 tokens, skewed popularity) plus a private suffix, served 64
    at a time, each then decoding 64 tokens.  Reports the prefix-cache hit
    rate, the fraction of prompt tokens whose prefill is skipped and the host
    cost per allocator call, for the product allocator and the oracle."""
    from paged_kv_cache_405_b200 import BlockAllocator
    n_req, conc, decode, bs, NB = args.requests, 64, 64, 16, 16384

    def workload():
        rng = np.random.default_rng(1234)
        prompts = [rng.integers(0, 32000, size=512).tolist() for _ in range(8)]
        w = 1.0 / np.arange(1, 9)
        reqs = []
        for _ in range(n_req):
            sys_p = prompts[int(rng.choice(8, p=w / w.sum()))]
            reqs.append(sys_p + rng.integers(0, 32000, size=int(rng.integers(16, 257))).tolist())
        return reqs, rng

    def simulate(alloc, limit=None):
        reqs, rng = workload()
        if limit is not None:
            reqs = reqs[:limit]
        live, nxt, calls, skipped, total = {}, 0, 0, 0, 0
        t0 = time.perf_counter()
        nr = len(reqs)
        while nxt < nr or live:
            while nxt < nr and len(live) < conc:
                st, nc, _ = alloc.seq_add_with_prompt(nxt, reqs[nxt])
                if st != 0:
                    raise RuntimeError("pool exhausted in the allocator benchmark")
                calls += 1
                skipped += nc
                total += len(reqs[nxt])
                live[nxt] = decode
                nxt += 1
            for sid in list(live):
                alloc.seq_append_tokens(sid, [int(rng.integers(0, 32000))])
                calls += 1
                live[sid] -= 1
                if live[sid] == 0:
                    alloc.seq_free(sid)
                    calls += 1
                    del live[sid]
        return time.perf_counter() - t0, calls, skipped, total

    prod = BlockAllocator(NB, bs, prefix_caching=True)
    t, calls, skipped, total = simulate(prod)
    cs = prod.cache_stats()
    # the oracle (snapshots its whole state per call) on a bounded sample,
    # with the product on the same sample for an exact counter comparison
    from oracle.allocator import CachingAllocator
    sample = min(n_req, 20)
    orc = CachingAllocator(NB, bs)
    t_o, calls_o, skipped_o, _ = simulate(orc, sample)
    prod2 = BlockAllocator(NB, bs, prefix_caching=True)
    _, _, skipped_p2, _ = simulate(prod2, sample)
    oc = orc.cache_stats()
    return {
        "metric": "prefix-cache hit rate and allocator host cost", "mode": "allocator-bench",
        "requests": n_req, "concurrency": conc, "decode_tokens": decode, "block_size": bs, "num_blocks": NB,
        "hit_rate": round(cs["hits"] / max(1, cs["lookups"]), 4),
        "prefill_tokens_skipped_frac": round(skipped / total, 4),
        "host_us_per_call": round(1e6 * t / calls, 3), "calls": calls, "evictions": cs["evictions"],
        "oracle": {"host_us_per_call": round(1e6 * t_o / calls_o, 3), "sample_requests": sample,
                   "same_counters_on_sample": (oc == prod2.cache_stats() and skipped_o == skipped_p2)},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1, help="GPUs (one rank each under torchrun; replicas, weak scaling)")
    ap.add_argument("--steps", type=int, default=20, help="timed decode steps")
    ap.add_argument("--warmup", type=int, default=5, help="untimed warm-up steps (at least 3)")
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(synth.CONFIGS),
                    help="headline workload (see synth.CONFIGS); default: the largest one-GPU decode workload")
    ap.add_argument("--targets", default="",
                    help="comma-separated workloads timed in the same run and reported under 'targets' "
                         "(default: %s when the headline is the default one; 'none' for none)"
                         % ",".join(DEFAULT_TARGETS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"],
                    help="ours: the CUDA library; reference: the CPU oracle on the host cores")
    ap.add_argument("--partition-size", type=int, default=0,
                    help="split-K partition in tokens (0: the workload's, else the library's choice)")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch size (small cases for profiling)")
    ap.add_argument("--prefix", type=int, default=0,
                    help="shared-prompt length of a shared-prefix workload (0: the workload's own)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg from host buffers")
    ap.add_argument("--e2e-in-flight", type=int, default=2,
                    help="steps in flight in the end-to-end leg (1: the host waits for each step's output "
                         "before it issues the next); the line also carries the 1-in-flight figure")
    ap.add_argument("--e2e-serial-output", action="store_true",
                    help="end-to-end leg: copy each step's output back on the kernels' stream (no output-copy "
                         "overlap), for comparison")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip timing the CPU oracle")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU-oracle sample length (all cores)")
    ap.add_argument("--reference-step-seconds", type=float, default=3.0,
                    help="CPU-oracle work per step of --impl reference")
    ap.add_argument("--allocator-bench", action="store_true",
                    help="host-only prefix-caching allocator simulation (prints its own JSON line)")
    ap.add_argument("--requests", type=int, default=2000, help="requests of --allocator-bench")
    ap.add_argument("--nvtx", action="store_true",
                    help="NVTX ranges around each step and each library call (e.g. for ncu --nvtx filters)")
    ap.add_argument("--clock-warm-s", type=float, default=0.5,
                    help="seconds of untimed repeats before the timed region, while clocks are sampled")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.allocator_bench:
        print(json.dumps(run_allocator_bench(args)), flush=True)
        return
    world, rank, local = dist_setup()
    if world != args.gpus and rank == 0:
        print("warning: --gpus %d but WORLD_SIZE %d" % (args.gpus, world), file=sys.stderr)
    if args.impl == "reference":
        line = run_reference(args, world, rank)
    else:
        line = run_ours(args, world, rank, local)
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
