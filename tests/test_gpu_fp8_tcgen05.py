"""The FP8 per-head decode built for the 5th-generation tensor cores
(tcgen05.mma kind::f8f6f4 reading the E4M3 K and V tiles from shared memory,
accumulators in tensor memory; build option PKV_FP8_TC=1) against the oracle.

The default build runs the same decode on mma.sync (measured faster on every
FP8 workload here), so this test builds the tcgen05 variant into a temporary
library and runs the FP8 decode parity tests through it in a child process
(the library is chosen when the binding is imported)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_tcgen05_fp8_decode_matches_oracle(tmp_path):
    import importlib.util
    spec = importlib.util.spec_from_file_location("_pkv_build", os.path.join(ROOT, "paged_kv_cache_405_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    lib = mod.build(defines=["PKV_FP8_TC=1"], out=str(tmp_path / "libpagedkv_tcgen05.so"))
    env = dict(os.environ, PKV_LIBRARY=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_gpu_fp8.py", "-q", "-p", "no:cacheprovider",
                        "-k", "decode or session"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "failed" not in r.stdout
