"""Build ``libpagedkv.so`` in-tree with nvcc for sm_100a (B200).

The CUDA kernels and the C ABI (``csrc/pagedkv.cu``) and the host allocator
(``csrc/allocator.cpp``) go into one shared library next to this file, so the
binary travels with the source tree.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libpagedkv.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

SOURCES = ["pagedkv.cu", "allocator.cpp"]
DEPS = SOURCES + ["common.cuh", "attention_common.cuh", "attention_simt.cuh", "attention_mma.cuh", "attention_fp8.cuh", "attention_fp8_tc.cuh", "prefix_tc.cuh",
                  "kv_append.cuh", "block_copy.cuh", "reduce.cuh"]

FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-Werror", "all-warnings",
         "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr", "-I", INCLUDE]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    srcs = [os.path.join(CSRC, f) for f in DEPS] + [os.path.join(INCLUDE, "pagedkv.h"), __file__]
    return any(os.path.getmtime(f) > t for f in srcs)


def build(force: bool = False, verbose: bool = False, defines=(), out: str = None) -> str:
    """Build the library (when stale, or always with force).  ``defines``
    (e.g. ["PKV_FP8_TC=1"]) select build-time options; ``out`` puts such a
    variant at another path, leaving the default library alone."""
    lib = out or LIB
    if not force and out is None and not defines and not _stale():
        return LIB
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [NVCC] + FLAGS + (["-Xptxas", "-v"] if verbose else []) + ["-D" + d for d in defines] + \
        [os.path.join(CSRC, f) for f in SOURCES] + ["-o", tmp]
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    # python build.py [--force] [-v] [-D NAME=VALUE ...] [-o PATH]
    args, defines, out = sys.argv[1:], [], None
    for i, a in enumerate(args):
        if a == "-D":
            defines.append(args[i + 1])
        elif a == "-o":
            out = args[i + 1]
    print(build(force="--force" in args, verbose="-v" in args, defines=defines, out=out))
