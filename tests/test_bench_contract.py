"""The benchmark's JSON line on the CPU: the reference arm (the oracle timed on the host
cores) prints one line with the keys the benchmark contract asks for, and under a
multi-rank launch only rank 0 prints it (the other ranks exit without work)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(args, env_extra=None):
    env = dict(os.environ)
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        env.pop(k, None)
    env.update(env_extra or {})
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT,
                         env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    return [json.loads(l) for l in res.stdout.splitlines() if l.startswith("{")]


@pytest.mark.parametrize("workload", ["tiny", "gpt2_bwd"])
def test_reference_arm_line(workload):
    lines = run_bench(["--impl", "reference", "--workload", workload, "--steps", "2",
                       "--warmup", "3", "--reference-budget-s", "4"])
    assert len(lines) == 1
    d = lines[0]
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 2
    assert d["higher_is_better"] is True and d["unit"] == "TFLOP/s"
    assert d["config"]["workload"] == workload
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == d["value"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(RANK="1", LOCAL_RANK="1", WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
               MASTER_PORT="29555")
    assert run_bench(["--impl", "reference", "--workload", "tiny", "--steps", "1",
                      "--warmup", "3", "--gpus", "2", "--reference-budget-s", "2"], env) == []


def test_warmup_below_three_is_rejected():
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl",
                          "reference", "--warmup", "2"], cwd=ROOT, capture_output=True,
                         text=True, timeout=120)
    assert res.returncode != 0 and "warmup" in res.stderr


def test_traffic_is_reported_only_for_the_kernel_it_was_measured_on(monkeypatch):
    """roofline.traffic comes from profiles/traffic.json only while the forward kernel's
    source hash matches the hash stored with the capture; otherwise it is null."""
    import io
    import bench
    stored = json.dumps({"long": {"kernel_source_sha": "abc", "dram_bytes_per_launch": 123}})
    monkeypatch.setattr(bench, "open", lambda path, *a, **k: io.StringIO(stored),
                        raising=False)
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: "abc")
    assert bench.profiled_traffic("long") == 123
    assert bench.profiled_traffic("gpt2") is None
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: "def")
    assert bench.profiled_traffic("long") is None
