"""The C-ABI library loads and exports every symbol include/pagedkv.h declares;
host-side validation rejects bad arguments before any launch (no GPU needed)."""
import ctypes
import os
import re

import pytest

import paged_kv_cache_405_b200 as pkv
from paged_kv_cache_405_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(pkv_\w+)\s*\(", src))
    return names


def test_header_declares_the_binding_exports():
    assert declared_symbols() == set(binding.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(binding.LIB_PATH)
    missing = [n for n in declared_symbols() if not hasattr(lib, n)]
    assert not missing


def test_status_strings():
    assert binding.lib.pkv_status_str(0) == b"ok"
    assert binding.lib.pkv_status_str(2) == b"no free block"


def test_workspace_size_rules():
    # fits one partition: no workspace
    assert pkv.attention_workspace_bytes(4, 4, 64, 512, 0) == 0
    # forced 512-token partitions of a 100k context
    # (8 seqs x 64 heads x 196 parts x (128+2) floats, then 8-byte split counters per row from a 256-byte boundary)
    parts = 8 * 64 * 196 * 130 * 4
    assert pkv.attention_workspace_bytes(8, 64, 128, 100_160, 512) == -(-parts // 256) * 256 + 8 * 64 * 8
    # the library's own partition: the whole context up to 512 tokens, else 512, for MHA and grouped queries
    assert pkv.attention_partition_size(8, 32, 32, 128, 500, 0) == 512
    assert pkv.attention_partition_size(8, 32, 32, 128, 8192, 0) == 512
    assert pkv.attention_partition_size(8, 32, 8, 128, 8192, 0) == 512
    assert pkv.attention_partition_size(8, 32, 8, 128, 8192, 1024) == 1024  # explicit sizes as given
    # the library's own choice is covered by the size it reports
    for hkv in (32, 8):
        auto = pkv.attention_partition_size(64, 32, hkv, 128, 8192, 0)
        assert pkv.attention_workspace_bytes(64, 32, 128, 8192, 0) >= pkv.attention_workspace_bytes(64, 32, 128, 8192, auto)
    auto = pkv.attention_partition_size(64, 32, 32, 128, 2048, 0)
    assert pkv.attention_workspace_bytes(64, 32, 128, 2048, 0) >= \
        pkv.attention_workspace_bytes(64, 32, 128, 2048, auto)


def host_only():
    """The validation tests below pass fake device pointers (address 16) and
    rely on every case being refused before a launch; where a GPU is present
    they are skipped, so that a case let through could never launch on them."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("host-validation test with fake device pointers")


def call_decode(**over):
    host_only()
    a = dict(out=16, q=16, k=16, v=16, bt=16, maxB=4, cl=16, S=1, Hq=4, Hkv=4, D=64, bs=16, NB=8,
             scale=0.0, P=0, ws=None, wsb=0, dt=1, stream=None)
    a.update(over)
    return binding.lib.pkv_paged_attention_decode(a["out"], a["q"], a["k"], a["v"], a["bt"], a["maxB"],
                                                  a["cl"], a["S"], a["Hq"], a["Hkv"], a["D"], a["bs"],
                                                  a["NB"], a["scale"], a["P"], a["ws"], a["wsb"], a["dt"],
                                                  a["stream"])


@pytest.mark.parametrize("over,status", [
    (dict(Hq=6, Hkv=4), binding.INVALID),          # group not integral
    (dict(bs=24), binding.INVALID),                # unsupported block size
    (dict(D=96), binding.UNSUPPORTED),
    (dict(dt=7), binding.INVALID),
    (dict(P=24), binding.INVALID),                 # not a multiple of 16
    (dict(q=8), binding.INVALID),                  # misaligned pointer
    (dict(out=None), binding.INVALID),
    (dict(maxB=64, P=16), binding.INVALID),        # split needs a workspace
    (dict(scale=-1.0), binding.INVALID),
    (dict(S=0, out=None), binding.OK),             # empty batch: nothing to do
])
def test_decode_validation(over, status):
    assert call_decode(**over) == status


@pytest.mark.parametrize("over,why", [
    (dict(S=65536), "at most 65535 sequences"),                       # one grid dimension
    (dict(maxB=65536, P=16), "too many partitions"),                  # 65536 partitions of 16 tokens
    (dict(maxB=(1 << 26) + 1), "max_blocks_per_seq*block_size too large"),   # over 2^30 tokens
    (dict(NB=1 << 25, Hkv=4, Hq=4, bs=16), "2^31 or more rows"),     # 32-bit TMA row coordinates
    (dict(Hq=65536, Hkv=4), "at most 65535 query heads"),             # keeps workspace sizes in range
])
def test_decode_size_limits_are_refused_before_any_launch(over, why):
    assert call_decode(**over) == binding.INVALID
    assert why in binding.lib.pkv_last_error().decode()


def call_decode_static(**over):
    host_only()
    a = dict(out=16, q=16, k=16, v=16, bt=16, maxB=4, cl=16, S=1, Hq=4, Hkv=4, D=64, bs=16, NB=8,
             scale=0.0, P=0, dt=1, stream=None)
    a.update(over)
    return binding.lib.pkv_paged_attention_decode_static(a["out"], a["q"], a["k"], a["v"], a["bt"], a["maxB"],
                                                         a["cl"], a["S"], a["Hq"], a["Hkv"], a["D"], a["bs"],
                                                         a["NB"], a["scale"], a["P"], a["dt"], a["stream"])


@pytest.mark.parametrize("over,why", [
    (dict(P=24), "partition_size must be 0 or a positive multiple of 16"),
    (dict(maxB=65536 * 2, P=16), "too many partitions"),
    (dict(bs=24), "block_size must be"),
    (dict(q=8), "16-byte aligned"),
])
def test_static_decode_reports_the_real_cause_before_the_scratch_size(over, why):
    """The built-in scratch is sized only once every other argument has
    passed, so a bad argument is named as such (no scratch message)."""
    assert call_decode_static(**over) == binding.INVALID
    msg = binding.lib.pkv_last_error().decode()
    assert why in msg and "scratch" not in msg


def test_static_decode_refuses_calls_beyond_its_scratch_before_any_launch():
    # 64 seqs x 32 heads x 128 partitions of 16 tokens x 130 floats > 64 MiB
    assert call_decode_static(S=64, Hq=32, Hkv=32, D=128, maxB=128, P=16) == binding.INVALID
    assert "split-K scratch" in binding.lib.pkv_last_error().decode()
    # an empty batch needs nothing and is accepted
    assert call_decode_static(S=0, out=None) == binding.OK


def test_workspace_queries_saturate_instead_of_wrapping():
    size_max = (1 << (8 * ctypes.sizeof(ctypes.c_size_t))) - 1
    big = (1 << 31) - 1
    assert pkv.attention_workspace_bytes(65535, big, 128, 1 << 30, 16) == size_max
    assert pkv.attention_shared_workspace_bytes(big, big, 128, 1 << 30, 16) == size_max
    assert pkv.attention_chunk_workspace_bytes(big, 65535, 128, 1 << 30, 16) == size_max
    # in range: the partials (2 x 3 rows x 4 parts x 66 floats), rounded up to 256 bytes, and a counter per row
    assert pkv.attention_workspace_bytes(2, 3, 64, 64, 16) == -(-(2 * 3 * 4 * 66 * 4) // 256) * 256 + 2 * 3 * 8


def test_append_and_copy_validation():
    host_only()
    lib = binding.lib
    # head_dim*elem not a multiple of 16 bytes
    assert lib.pkv_kv_append(16, 16, 16, 16, 16, 1, 4, 1, 6, 16, 1, None) == binding.INVALID
    assert lib.pkv_kv_append(None, None, None, None, None, 0, 4, 1, 64, 16, 1, None) == binding.OK
    assert lib.pkv_block_copy(16, 16, 16, -1, 4, 1, 64, 16, 1, None) == binding.INVALID
    assert lib.pkv_block_copy(None, None, None, 0, 4, 1, 64, 16, 1, None) == binding.OK


def test_device_calls_demand_cuda_tensors():
    import torch
    k = torch.zeros(4, 1, 16, 64)
    with pytest.raises(TypeError):
        pkv.kv_append(k[0], k[0], k, k, torch.zeros(1, dtype=torch.int64))


def test_package_exposes_every_binding_call():
    import inspect
    public = [n for n, f in inspect.getmembers(binding, inspect.isfunction)
              if not n.startswith("_") and f.__module__ == binding.__name__]
    missing = [n for n in public if not hasattr(pkv, n)]
    assert not missing


def test_build_runs_from_a_checkout_without_the_library(tmp_path):
    """build() must not import the package (whose __init__ loads the library)
    before it has compiled it: a fresh checkout has no libpagedkv.so."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("import sys, __graft_entry__ as g\n"
            "m = g._load_by_path('_b', g.os.path.join(g.ROOT, 'paged_kv_cache_405_b200', 'build.py'))\n"
            "assert callable(m.build)\n"
            "assert 'paged_kv_cache_405_b200' not in sys.modules\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr


def test_nvtx_ranges_name_the_entry_point_and_always_close(monkeypatch):
    """With NVTX on, each device call opens a range named after its C entry
    point and closes it even when the call raises (here: CPU tensors)."""
    import torch
    events = []
    monkeypatch.setattr(torch.cuda.nvtx, "range_push", lambda name: events.append(("push", name)))
    monkeypatch.setattr(torch.cuda.nvtx, "range_pop", lambda: events.append(("pop",)))
    k = torch.zeros(4, 2, 16, 64, dtype=torch.bfloat16)
    new = torch.zeros(1, 2, 64, dtype=torch.bfloat16)
    pkv.set_nvtx(True)
    try:
        with pytest.raises((ValueError, TypeError)):
            pkv.kv_append(new, new, k, k, torch.zeros(1, dtype=torch.int64))
        with pytest.raises((ValueError, TypeError)):
            pkv.block_copy(k, k, torch.zeros(1, 2, dtype=torch.int32))
    finally:
        pkv.set_nvtx(False)
    assert events == [("push", "pkv_kv_append"), ("pop",), ("push", "pkv_block_copy"), ("pop",)]
    pkv.set_nvtx(False)
    with pytest.raises((ValueError, TypeError)):   # off: no ranges
        pkv.kv_append(new, new, k, k, torch.zeros(1, dtype=torch.int64))
    assert len(events) == 4


def test_binding_rejects_inconsistent_buffers():
    """The C calls see pointers and sizes only: the binding rejects tensors
    whose sizes or element types disagree with the sizes it passes, each of
    which would make a kernel read or write past a buffer."""
    import torch
    bf, f32, u8 = torch.bfloat16, torch.float32, torch.uint8
    k = torch.zeros(8, 2, 16, 64, dtype=bf)
    q = torch.zeros(3, 4, 64, dtype=bf)
    bt = torch.zeros(3, 5, dtype=torch.int32)
    cl = torch.zeros(3, dtype=torch.int32)
    new = torch.zeros(2, 2, 64, dtype=bf)
    sm = torch.zeros(2, dtype=torch.int64)
    # consistent arguments pass
    binding._check_pools(k, k.clone())
    binding._check_attention(q.clone(), q, k, bt, cl, 3, pool_type=True)
    binding._check_attention(q.clone(), q, k.to(u8), bt, cl, 3, pool_type=False)   # FP8 pools
    binding._check_new(new, new.clone(), k, sm, pool_type=True)
    binding._check_new(new.float(), new.float(), k.to(u8), sm, pool_type=False)   # FP8 append converts
    bad = [
        lambda: binding._check_pools(k, k[:4].clone()),                                   # V pool smaller
        lambda: binding._check_pools(k, k.float()),                                       # V pool wider type
        lambda: binding._check_pools(k[0], k[0]),                                         # not 4-D
        lambda: binding._check_attention(q.float(), q, k, bt, cl, 3, pool_type=True),     # out wider than q
        lambda: binding._check_attention(q[:2].clone(), q, k, bt, cl, 3, pool_type=True),  # out smaller
        lambda: binding._check_attention(q.float(), q.float(), k, bt, cl, 3, pool_type=True),   # q vs pools
        lambda: binding._check_attention(q[..., :32].clone(), q[..., :32].clone(), k, bt, cl, 3, pool_type=True),
        lambda: binding._check_attention(q.clone(), q, k, bt[:2], cl, 3, pool_type=True),  # table rows
        lambda: binding._check_attention(q.clone(), q, k, bt, cl[:2], 3, pool_type=True),  # lengths
        lambda: binding._check_new(new, new, k, sm[:1], pool_type=True),                  # one slot short
        lambda: binding._check_new(new.float(), new.float(), k, sm, pool_type=True),      # wider than pool
        lambda: binding._check_new(new, new.float(), k, sm, pool_type=True),              # K / V differ
        lambda: binding._check_new(torch.zeros(2, 4, 64, dtype=bf), torch.zeros(2, 4, 64, dtype=bf), k, sm,
                                   pool_type=True),                                       # kv heads
    ]
    for i, call in enumerate(bad):
        with pytest.raises((ValueError, TypeError)):
            call()
            raise AssertionError("case %d passed" % i)


def call_chunk(**over):
    host_only()
    a = dict(out=16, q=16, k=16, v=16, bt=16, maxB=4, cl=16, qs=16, S=1, T=2, mq=2, Hq=4, Hkv=4, D=64, bs=16,
             NB=8, scale=0.0, P=0, ws=None, wsb=0, dt=1, stream=None)
    a.update(over)
    return binding.lib.pkv_paged_attention_chunk(a["out"], a["q"], a["k"], a["v"], a["bt"], a["maxB"], a["cl"],
                                                 a["qs"], a["S"], a["T"], a["mq"], a["Hq"], a["Hkv"], a["D"],
                                                 a["bs"], a["NB"], a["scale"], a["P"], a["ws"], a["wsb"], a["dt"],
                                                 a["stream"])


@pytest.mark.parametrize("over,status,why", [
    (dict(dt=0), binding.UNSUPPORTED, "16-bit element types only"),
    (dict(Hq=64, Hkv=2), binding.INVALID, "1..16 times num_kv_heads"),
    (dict(mq=0), binding.INVALID, "sizes must be positive"),
    (dict(qs=None), binding.INVALID, "null pointer"),
    (dict(maxB=4096, P=16, mq=512, Hq=8, Hkv=1), binding.INVALID, "row tiles x partitions"),
    (dict(S=0, out=None), binding.OK, ""),
])
def test_chunk_validation(over, status, why):
    assert call_chunk(**over) == status
    assert why in binding.lib.pkv_last_error().decode()


def test_fp8_calls_validation():
    host_only()
    lib = binding.lib

    def append(**over):
        a = dict(T=1, D=64, src=1, ks=1.0, vs=1.0)
        a.update(over)
        return lib.pkv_kv_append_fp8(16, 16, 16, 16, 16, a["T"], 4, 1, a["D"], 16, a["src"], a["ks"], a["vs"], None)

    assert append(ks=0.0) == binding.INVALID and "positive and finite" in lib.pkv_last_error().decode()
    assert append(vs=float("inf")) == binding.INVALID
    assert append(D=72) == binding.INVALID and "multiple of 16" in lib.pkv_last_error().decode()
    assert append(src=binding.FP8_E4M3) == binding.INVALID                  # new K/V are 16- or 32-bit

    def decode(**over):
        a = dict(dt=1, ks=1.0, vs=1.0)
        a.update(over)
        return lib.pkv_paged_attention_decode_fp8(16, 16, 16, 16, 16, 4, 16, 1, 4, 4, 64, 16, 8, 0.0, a["ks"],
                                                  a["vs"], 0, None, 0, a["dt"], None)

    assert decode(dt=0) == binding.UNSUPPORTED                              # fp32 q/out
    assert decode(ks=-1.0) == binding.INVALID and "positive and finite" in lib.pkv_last_error().decode()


def test_workspace_queries_cover_every_call_random():
    """For random shapes, the size each workspace query reports holds the
    partials the call writes under the partition size the library picks:
    (rows) x (partitions, + 1 slot in shared-prefix mode) x (D + 2) floats
    whenever a context spans more than one partition, and in shared-prefix
    mode 8 bytes per sequence of membership after them."""
    import numpy as np
    rng = np.random.default_rng(0)
    for _ in range(2000):
        S, Hq = int(rng.integers(1, 300)), int(rng.choice([1, 8, 32, 64]))
        D = int(rng.choice([64, 128]))
        max_len = int(rng.integers(1, 4096)) * int(rng.choice([16, 64, 256]))
        P = int(rng.choice([0, 0, 16, 64, 256, 512, 1024]))
        eff = pkv.attention_partition_size(S, Hq, 1, D, max_len, P)
        assert eff > 0 and eff % 16 == 0 and (P == 0 or eff == P)
        nparts = -(-max_len // eff)
        per = Hq * (D + 2) * 4
        ws = pkv.attention_workspace_bytes(S, Hq, D, max_len, P)
        assert ws >= (S * nparts * per if nparts > 1 else 0)
        assert pkv.attention_shared_workspace_bytes(S, Hq, D, max_len, P) >= S * (nparts + 1) * per + 8 * S
        T = S * int(rng.integers(1, 5))
        cw = pkv.attention_chunk_workspace_bytes(T, Hq, D, max_len, P)
        assert cw >= (T * nparts * per if nparts > 1 else 0)


def test_plain_c_consumer_builds_and_runs(tmp_path):
    """The header compiles as C99 with warnings as errors, a C program links
    the library, and its host-only calls (allocator on the pages' worked
    example, fork and copy-on-write, exhaustion, queries, an empty batch)
    behave as documented."""
    import subprocess
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(binding.LIB_PATH)
    exe = str(tmp_path / "host_calls")
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(root, "include"),
                           "-o", exe, os.path.join(root, "tests", "c_abi", "host_calls.c"), "-L", libdir,
                           "-l:" + os.path.basename(binding.LIB_PATH), "-Wl,-rpath," + libdir])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr


def test_step_struct_layout_matches_the_header(tmp_path):
    """The binding's ctypes pkv_step / pkv_copy have the header's size and
    field offsets (a C program compiled against the header prints them)."""
    import subprocess
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    fields = [f for f, _ in binding.PkvStep._fields_]
    cnames = ["in" if f == "in_" else f for f in fields]
    src = ["#include <stddef.h>", "#include <stdio.h>", '#include "pagedkv.h"', "int main(void) {",
           '  printf("%zu %zu\\n", sizeof(pkv_step), sizeof(pkv_copy));',
           '  printf("%zu %zu %zu\\n", offsetof(pkv_copy, dst), offsetof(pkv_copy, src), offsetof(pkv_copy, bytes));']
    src += ['  printf("%%zu\\n", offsetof(pkv_step, %s));' % c for c in cnames]
    src += ["  return 0;", "}"]
    c = tmp_path / "layout.c"
    c.write_text("\n".join(src) + "\n")
    exe = str(tmp_path / "layout")
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(root, "include"), "-o", exe,
                           str(c)])
    out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split()
    assert int(out[0]) == ctypes.sizeof(binding.PkvStep) and int(out[1]) == ctypes.sizeof(binding.PkvCopy)
    assert [int(x) for x in out[2:5]] == [binding.PkvCopy.dst.offset, binding.PkvCopy.src.offset,
                                          binding.PkvCopy.bytes.offset]
    assert [int(x) for x in out[5:]] == [getattr(binding.PkvStep, f).offset for f in fields]


def step_struct(**over):
    st = binding.PkvStep(struct_size=ctypes.sizeof(binding.PkvStep), kind=binding.STEP_DECODE, num_blocks=8,
                         num_kv_heads=4, head_dim=64, block_size=16, dtype=1, k_scale=1.0, v_scale=1.0,
                         max_blocks_per_seq=4, num_q_heads=4)
    for k, v in over.items():
        setattr(st, k, v)
    return st


@pytest.mark.parametrize("over,why", [
    (dict(struct_size=8), "struct_size"),
    (dict(kind=7), "bad kind"),
    (dict(n_in=-1), "bad copy lists"),
    (dict(n_out=2), "bad copy lists"),                      # no list given
    (dict(num_tokens=-3), "counts must be >= 0"),
    (dict(copy_stream=16), "go together"),                  # overlapped copies: stream without its events
    (dict(inputs_free=16, inputs_ready=32), "go together"),  # events without the stream
    (dict(out_stream=16), "go together"),                   # overlapped output copies: stream without its event
    (dict(out_stream=16, outputs_done=32), "needs copy_stream"),  # ... without the overlapped input copies
    (dict(num_pairs=1, pairs=16, k_pool=16, v_pool=8), "16-byte aligned"),        # pkv_block_copy's own check
    (dict(num_tokens=2, k_new=16, v_new=16, k_pool=16, v_pool=16, slot_mapping=16, head_dim=6), "multiple of 16"),
    (dict(num_seqs=1, q=16, attn_out=16, k_pool=16, v_pool=16, block_tables=16, context_lens=16, num_q_heads=6),
     "multiple of num_kv_heads"),                             # the attention call's own check
])
def test_step_from_host_refuses_bad_steps(over, why):
    host_only()
    assert binding.lib.pkv_step_from_host(ctypes.byref(step_struct(**over)), None) == binding.INVALID
    assert why in binding.lib.pkv_last_error().decode()


def test_step_from_host_empty_step_and_null():
    host_only()
    assert binding.lib.pkv_step_from_host(ctypes.byref(step_struct()), None) == binding.OK   # nothing to do
    assert binding.lib.pkv_step_from_host(None, None) == binding.INVALID


def test_last_error_is_per_thread():
    """pkv_last_error() describes the last failed call on the calling thread:
    two threads failing different calls concurrently each read their own
    message (ctypes releases the GIL inside the calls)."""
    import threading
    lib = binding.lib
    results = {}

    def worker(name, call, expect):
        ok = True
        for _ in range(2000):
            call()
            ok &= expect in lib.pkv_last_error().decode()
        results[name] = ok

    a = threading.Thread(target=worker, args=("append", lambda: lib.pkv_kv_append(
        None, None, None, None, None, -1, 4, 1, 64, 16, 1, None), "pkv_kv_append"))
    b = threading.Thread(target=worker, args=("alloc", lambda: lib.pkv_alloc_create(0, 16, None),
                                               "pkv_alloc_create"))
    a.start()
    b.start()
    a.join()
    b.join()
    assert results == {"append": True, "alloc": True}


def test_build_tracks_every_source_and_targets_sm100a():
    """Every CUDA/C++ source and header of the library is a build dependency
    (an edit rebuilds the library), and the build targets sm_100a only."""
    import importlib.util
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("_b", os.path.join(root, "paged_kv_cache_405_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    files = {f for f in os.listdir(b.CSRC) if f.endswith((".cu", ".cuh", ".cpp", ".h"))}
    assert files <= set(b.DEPS), files - set(b.DEPS)
    i = b.FLAGS.index("-gencode")
    assert b.FLAGS[i + 1] == "arch=compute_100a,code=sm_100a" and b.FLAGS.count("-gencode") == 1
    assert "-lineinfo" in b.FLAGS


def test_product_and_oracle_import_nothing_of_each_other():
    """The product package loads no part of the oracle and the oracle loads no
    part of the product (fresh interpreters), and no product source names it."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("import sys, {mod}\n"
            "bad = [m for m in sys.modules if m == {other!r} or m.startswith({other!r} + '.')]\n"
            "assert not bad, bad\n")
    for mod, other in (("paged_kv_cache_405_b200", "oracle"), ("oracle", "paged_kv_cache_405_b200")):
        r = subprocess.run([sys.executable, "-c", code.format(mod=mod, other=other)], cwd=root,
                           capture_output=True, text=True, timeout=120)
        assert r.returncode == 0, r.stderr[-2000:]
    pkg = os.path.join(root, "paged_kv_cache_405_b200")
    for dirpath, _, names in os.walk(pkg):
        for n in names:
            if n.endswith((".py", ".cu", ".cuh", ".cpp", ".h")):
                text = open(os.path.join(dirpath, n), encoding="utf-8").read()
                assert "import oracle" not in text and "from oracle" not in text and "oracle.c" not in text, n
