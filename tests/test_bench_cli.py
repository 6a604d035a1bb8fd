"""bench.py's command-line contract, on the CPU: the reference arm (the fp64 oracle timed
on host cores) prints one JSON line with the contract's keys; under a multi-rank launch
only rank 0 prints; fewer than 3 warm-up steps are refused; the CPU baseline reports the
oracle on all host cores and on one thread."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e")


def _bench(*args, env=None):
    e = dict(os.environ)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True,
                          text=True, env=e, timeout=600)


def test_reference_arm_prints_one_contract_line():
    r = _bench("--impl", "reference", "--steps", "3", "--warmup", "3", "--config", "tiny_f32_T64_n4_d64")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in KEYS:
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 3 and d["warmup"] == 3 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "tiny_f32_T64_n4_d64"


def test_reference_arm_other_ranks_exit_quietly():
    r = _bench("--impl", "reference", "--gpus", "2", "--steps", "3", "--warmup", "3",
               "--config", "tiny_f32_T64_n4_d64", env={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_too_few_warmup_steps_are_refused():
    r = _bench("--warmup", "2")
    assert r.returncode != 0 and "--warmup must be >= 3" in r.stderr


def test_cpu_baseline_reports_all_cores_and_one_thread():
    sys.path.insert(0, ROOT)
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    from mhc_hyper_connections_b200 import workloads as wl
    w = wl.make_config("tiny_f32_T64_n4_d64")
    cb = bench.cpu_baseline(w, seconds=0.2, chunk=16, single_seconds=0.1)
    assert cb["kind"] == "oracle" and cb["unit"] == "tokens/s" and cb["value"] > 0 and cb["cores"] >= 1
    one = cb["single_thread"]
    assert one["cores"] == 1 and one["value"] > 0 and "one thread" in one["sample"]
    json.dumps(cb)
