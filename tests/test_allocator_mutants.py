"""The allocator tests catch plausible mistakes in the product's C++
allocator: each case plants one mistake in a copy of ``allocator.cpp``,
links it with the library's CUDA object into a separate library (the
package loads it through PKV_LIBRARY) and runs the host allocator tests
against it, which must fail.  The mistakes live only in temporary copies."""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "paged_kv_cache_405_b200", "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]

# name: (text in allocator.cpp, replacement)
MUTANTS = {
    "no copy-on-write": ("bool must_copy(int32_t b) const { return ref[b] > 1 || node_of[b] >= 0; }",
                         "bool must_copy(int32_t b) const { return false && b; }"),
    "cached blocks written in place": ("bool must_copy(int32_t b) const { return ref[b] > 1 || node_of[b] >= 0; }",
                                       "bool must_copy(int32_t b) const { return ref[b] > 1; }"),
    "freed blocks to the front": ("            free_q.push_back(b);\n", "            free_q.push_front(b);\n"),
    "newest evicted first": ("        int32_t b = lru.front();\n        lru.pop_front();",
                             "        int32_t b = lru.back();\n        lru.pop_back();"),
    "fork without refcounts": ("    for (int32_t b : c.table) a->ref[b] += 1;\n", ""),
    "failures not counted": ("        a->alloc_failures += 1;\n        set_error(\"pkv_seq_append_slots: free pool exhausted\");",
                             "        set_error(\"pkv_seq_append_slots: free pool exhausted\");"),
    "batched dry run ignores cached blocks": ("if (holders > 1 || a->node_of[b] >= 0) {", "if (holders > 1) {"),
    "batched dry run ignores a released original": ("                if (holders == 1) avail += 1;", ""),
    "single call ignores a released original": ("else avail += (a->ref[s.table[L / bs]] == 1) ? 0 : -1;",
                                                "else avail -= 1;"),
    "cache key without its parent": ("        CacheKey k{s.chain, s.tail};", "        CacheKey k{kRoot, s.tail};"),
}
TESTS = ["tests/test_allocator.py", "tests/test_prefix_cache.py", "tests/test_session_host.py"]


def _build_and_run(d, obj, name):
    old, new = MUTANTS[name]
    src = open(os.path.join(CSRC, "allocator.cpp")).read()
    if src.count(old) != 1:
        return "the planted mistake must replace exactly one place"
    tag = "m%d" % list(MUTANTS).index(name)
    cpp, mobj, lib = (os.path.join(d, tag + ".cpp"), os.path.join(d, tag + ".o"),
                      os.path.join(d, "libpagedkv_%s.so" % tag))
    mutant = src.replace(old, new).replace('#include "../../include/pagedkv.h"', '#include "pagedkv.h"')
    open(cpp, "w").write(mutant)
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-I", os.path.join(ROOT, "include"), "-c", cpp,
                           "-o", mobj])
    subprocess.check_call([NVCC, "-shared", *ARCH, obj, mobj, "-o", lib])
    r = subprocess.run([sys.executable, "-m", "pytest", *TESTS, "-x", "-q", "-m", "not gpu", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=dict(os.environ, PKV_LIBRARY=lib), capture_output=True, text=True, timeout=900)
    if r.returncode == 0:
        return "no test caught it"
    if "failed" not in r.stdout:
        return r.stdout[-2000:] + r.stderr[-2000:]
    return None


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    """Build every mutant library and run the allocator tests against each,
    the runs side by side (they are independent processes)."""
    from concurrent.futures import ThreadPoolExecutor
    d = str(tmp_path_factory.mktemp("allocator_mutants"))
    obj = os.path.join(d, "pagedkv.o")
    subprocess.check_call([NVCC, "-O3", "-std=c++17", *ARCH, "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
                           "-I", os.path.join(ROOT, "include"), "-c", os.path.join(CSRC, "pagedkv.cu"), "-o", obj])
    with ThreadPoolExecutor(max_workers=max(2, min(len(MUTANTS), os.cpu_count() or 2))) as ex:
        futures = {name: ex.submit(_build_and_run, d, obj, name) for name in MUTANTS}
        return {name: f.result() for name, f in futures.items()}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_allocator_tests_catch_planted_mistake(name, outcomes):
    assert outcomes[name] is None, "%s: %s" % (name, outcomes[name])
