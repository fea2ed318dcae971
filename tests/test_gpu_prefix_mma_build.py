"""The shared-prefix pass built as mma.sync tiles (build option
PKV_PREFIX_TC=0; the default library runs the pass on tcgen05 at head_dim 128,
and head_dim 64 always uses mma.sync) against the oracle: the library is built
with the option into a temporary file and the shared-prefix parity tests --
small groups, groups of more than 128 rows, and the full-size shared-prompt
decode step -- run through it in a child process (the library is chosen when
the binding is imported)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_mma_sync_prefix_pass_matches_oracle(tmp_path):
    import importlib.util
    spec = importlib.util.spec_from_file_location("_pkv_build", os.path.join(ROOT, "paged_kv_cache_405_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    lib = mod.build(defines=["PKV_PREFIX_TC=0"], out=str(tmp_path / "libpagedkv_prefix_mma.so"))
    env = dict(os.environ, PKV_LIBRARY=lib)
    files = ["tests/test_gpu_shared_prefix.py", "tests/test_gpu_prefix_cache.py", "tests/test_gpu_fullsize.py"]
    r = subprocess.run([sys.executable, "-m", "pytest", *files, "-k", "not fullsize or llama13b_prefix", "-q",
                        "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "failed" not in r.stdout
