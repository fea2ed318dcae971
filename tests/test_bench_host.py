"""Host-side logic of bench.py on CPU tensors: allocator replay of each
workload's layout, step planning (beams, copy-on-write), byte accounting, and
the multi-rank reductions over a 2-rank gloo group."""
import os

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import bench
import oracle
import synth


@pytest.mark.parametrize("cfg,over", [
    ("tiny", {}),
    ("llama7b", dict(S=6, Hq=2, Hkv=2, D=64)),
    ("llama13b_prefix", dict(S=5, Hq=1, Hkv=1, D=64)),
    ("llama3_gqa_bs32", dict(S=3, Hq=4, Hkv=1, D=64, len_fixed=300)),
    ("longctx_beam", dict(S=2, Hq=2, Hkv=1, D=64, len_fixed=1000)),
    ("spec_verify", dict(S=3, Hq=4, Hkv=1, D=64, len_uniform=(20, 300))),
    ("llama7b_fp8", dict(S=4, Hq=2, Hkv=2, D=64)),
])
def test_workload_steps_on_cpu(cfg, over):
    sh = synth.shrink(synth.CONFIGS[cfg], **over)
    wl = bench.Workload(sh, sh.seed, "cpu", 0)
    orc = oracle.Allocator(wl.batch.num_blocks, sh.bs, wl.batch.free_order)
    lens0 = wl.batch.lens.copy()
    for i in range(3):
        p = wl.plan()
        step = max(1, sh.chunk)
        assert p.lens.tolist() == (lens0 + step * (i + 1)).tolist()
        T = sh.S * max(1, sh.beams, sh.chunk)
        assert len(p.slot_mapping) == T and len(set(p.slot_mapping.tolist())) == T
        if sh.beams:
            assert len(p.cow_pairs) == sh.S * (sh.beams - 1) or i > 0
        else:
            assert len(p.cow_pairs) == 0
        total, a = wl.step_bytes(p)
        assert a["kv"] <= a["logical_kv"] and total > a["kv"]
    del orc


def test_attention_bytes_counts_shared_blocks_once():
    bt = np.array([[5, 6, 1], [5, 6, 2]], np.int32)
    lens = np.array([40, 35])
    a = bench.attention_bytes(bt, lens, Hq=1, Hkv=1, D=8, bs=16, elt=2, P=512)
    # blocks 5, 6 once (32 tokens) + block 1 (8 tokens) + block 2 (3 tokens)
    assert a["kv"] == 2 * 8 * 2 * (32 + 8 + 3)
    assert a["logical_kv"] == 2 * 8 * 2 * 75 and a["ws"] == 0
    # KV memory utilisation: 43 tokens held in 4 physical blocks of 16 slots
    assert a["kv_util"] == 43 / 64


def _ranks(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    mx = bench.max_over_ranks(float(rank + 1), world)
    sm = bench.sum_over_ranks(float(rank + 1), world)
    bench.barrier(world)
    q.put((rank, mx, sm))
    torch.distributed.destroy_process_group()


def test_rank_reductions_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    ps = [ctx.Process(target=_ranks, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
    assert res == [(0, 2.0, 3.0), (1, 2.0, 3.0)]


def test_cpu_baseline_sample_runs_on_one_thread():
    b = synth.make_batch(synth.CONFIGS["tiny"])
    v, sps, desc, secs = bench.oracle_sample(b, 0.05, threads=1)
    assert v > 0 and sps > 0 and secs >= 0.05 and "1 threads" in desc
    assert isinstance(bench.cpu_model(), str) and bench.cpu_model()


def test_reference_arm_prints_one_contract_line():
    """``bench.py --impl reference`` (the CPU oracle on the host cores) prints
    one JSON line with the contract's keys, its own cpu_baseline and an e2e
    object without host<->device bytes."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "tiny", "--steps", "2",
                        "--warmup", "3", "--reference-step-seconds", "0.5"], cwd=root, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["config"]["workload"] == "tiny" and d["value"] > 0 and d["higher_is_better"] is True
    import argparse
    sh = bench.workload_shape(argparse.Namespace(config="tiny", batch=0, warmup=3, steps=2))
    assert d["config"]["batch"] == sh.S and d["config"]["head_dim"] == sh.D and d["config"]["block_size"] == sh.bs
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_both_arms_name_the_same_config():
    """The reference arm's ``config`` is built by the same function from the
    same seeded batch as this arm's, so the two lines name one workload
    (shape keys included)."""
    import argparse
    args = argparse.Namespace(config="llama7b", batch=0, partition_size=0, warmup=5, steps=20)
    sh = bench.workload_shape(args)
    a = bench.workload_config("llama7b", sh, synth.make_batch(sh, device="cpu"), args, 1)
    b = bench.workload_config("llama7b", sh, synth.make_batch(sh, device="cpu", seed=sh.seed), args, 1)
    assert a == b
    for key in ("workload", "batch", "q_heads", "kv_heads", "head_dim", "block_size", "partition_size",
                "mean_context", "l2", "parallelism"):
        assert key in a, key
    assert a["batch"] == 64 and a["q_heads"] == 32 and a["head_dim"] == 128 and a["block_size"] == 16


def test_default_run_times_the_largest_config_and_the_targets():
    import argparse
    assert bench.DEFAULT_CONFIG == "llama3_gqa_bs16"
    big = max((s.S * s.Hkv * (s.len_fixed or 0), n) for n, s in synth.CONFIGS.items() if not s.kv_fp8)
    assert big[1].startswith("llama3_gqa")
    ns = argparse.Namespace(targets="", batch=0, config=bench.DEFAULT_CONFIG)
    assert bench.target_names(ns) == ["llama13b_prefix", "longctx_beam", "llama7b"]
    assert bench.target_names(argparse.Namespace(targets="", batch=64, config=bench.DEFAULT_CONFIG)) == []
    assert bench.target_names(argparse.Namespace(targets="", batch=0, config="llama7b")) == []
    assert bench.target_names(argparse.Namespace(targets="none", batch=0, config=bench.DEFAULT_CONFIG)) == []
    assert bench.target_names(argparse.Namespace(targets="tiny,llama7b", batch=8, config="tiny")) == \
        ["tiny", "llama7b"]


def test_warmup_below_three_is_refused():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2", "--impl", "reference", "--config", "tiny"])


def fake_smi(tmp_path, lines):
    """A stand-in nvidia-smi: prints the given sample lines, leaves a marker
    file once they are out, then waits to be stopped."""
    d = tmp_path / "bin"
    d.mkdir(exist_ok=True)
    exe = d / "nvidia-smi"
    marker = tmp_path / "printed"
    if marker.exists():
        marker.unlink()
    exe.write_text("#!/bin/sh\n" + "".join("echo '%s'\n" % ln for ln in lines) +
                   "touch '%s'\nexec sleep 30\n" % marker)
    exe.chmod(0o755)
    return str(d)


def wait_printed(tmp_path):
    import time
    t0 = time.time()
    while not (tmp_path / "printed").exists():
        assert time.time() - t0 < 30, "the stand-in nvidia-smi never ran"
        time.sleep(0.02)


def test_clock_sampler_reports_median_max_and_active_reasons(tmp_path, monkeypatch):
    """The clocks object of the bench line from nvidia-smi samples (index,
    SM clock, max SM clock, power, reason mask, then hw_slowdown,
    hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap): median SM clock,
    max clock, every reason seen active, sample count; other lines ignored."""
    monkeypatch.setenv("PATH", fake_smi(tmp_path, [
        "0, 1965, 1965, 700.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1950, 1965, 710.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1980, 1965, 690.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, [N/A], 1965, 690.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]) + os.pathsep + os.environ["PATH"])
    c = bench.ClockSampler(0)
    c.start()
    wait_printed(tmp_path)
    assert c.stop() == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}

    monkeypatch.setenv("PATH", fake_smi(tmp_path, [
        "0, 1400, 1965, 990.0, 0x0000000000000008, Active, Not Active, Not Active, Not Active",
        "0, 1500, 1965, 990.0, 0x0000000000000020, Not Active, Active, Not Active, Active",
    ]) + os.pathsep + os.environ["PATH"])
    c = bench.ClockSampler(0)
    c.start()
    wait_printed(tmp_path)
    got = c.stop()
    assert got["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap"] and got["sm_mhz"] == 1450.0


def test_clock_sampler_without_nvidia_smi_reports_nothing(tmp_path, monkeypatch):
    empty = tmp_path / "empty"
    empty.mkdir()
    monkeypatch.setenv("PATH", str(empty))
    c = bench.ClockSampler(0)
    c.start()
    assert c.stop() is None


def test_roofline_peak_and_traffic_lookups(tmp_path, monkeypatch):
    """The peak comes from MEASURED_PEAKS.json (else the 6.65 TB/s fallback);
    recorded DRAM traffic is reported only for entries taken on the current
    kernel sources (their hash), else null."""
    import json
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_hbm_peak() == (6650.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6545.3, "bf16_tflops": 1590}))
    assert bench.measured_hbm_peak() == (6545.3, "measured")

    csrc = tmp_path / "paged_kv_cache_405_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("__global__ void k() {}\n")
    (tmp_path / "profiles").mkdir()
    h = bench.kernel_source_hash()
    (tmp_path / "profiles" / "dram_traffic.txt").write_text(
        "# workload hash bytes note\nllama7b %s 1132961280 note\nllama7b 0000000000000000 1 stale\n" % h)
    assert bench.recorded_traffic("llama7b") == 1132961280.0
    assert bench.recorded_traffic("llama13b_prefix") is None
    (csrc / "k.cu").write_text("__global__ void k() { }\n")      # the kernel changed: the entry is stale
    assert bench.kernel_source_hash() != h and bench.recorded_traffic("llama7b") is None


def test_allocator_bench_line():
    """--allocator-bench (host only): one JSON line with the prefix-cache
    hit rate and host cost, and the product's counters equal the oracle's on
    a sample of the same requests."""
    import argparse
    d = bench.run_allocator_bench(argparse.Namespace(requests=60))
    assert d["mode"] == "allocator-bench" and d["requests"] == 60
    assert 0.5 < d["hit_rate"] <= 1.0 and 0.5 < d["prefill_tokens_skipped_frac"] <= 1.0
    assert d["host_us_per_call"] > 0 and d["calls"] > 0
    assert d["oracle"]["same_counters_on_sample"] is True


def test_prefix_override_reaches_the_headline_workload_only():
    import argparse
    ns = argparse.Namespace(config="llama13b_prefix", batch=0, prefix=4096, warmup=3, steps=5, targets="")
    assert bench.workload_shape(ns).prefix == 4096
    assert bench.workload_shape(ns, "llama13b_prefix").prefix == 4096      # the headline, named as measured
    ns2 = argparse.Namespace(config="llama3_gqa_bs16", batch=0, prefix=4096, warmup=3, steps=5, targets="")
    assert bench.workload_shape(ns2, "llama13b_prefix").prefix == synth.CONFIGS["llama13b_prefix"].prefix
    assert bench.workload_shape(ns2).prefix == 0                            # no shared prompt to override
