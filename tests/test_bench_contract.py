"""bench.py's reference arm on CPU: one JSON line with the contract's keys.

`--impl reference` times the CPU oracle (no GPU needed), so its output can be
checked here: exactly one line on stdout, the metric / unit / direction of
the CUDA arm, a cpu_baseline describing the run, an e2e object with no host
copies, and non-zero ranks of a multi-rank launch exiting quietly.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_one_contract_line():
    res = run_bench(["--impl", "reference", "--steps", "2", "--warmup", "1"])
    assert res.returncode == 0, res.stderr
    lines = [ln for ln in res.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, res.stdout
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["unit"] == "GB/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["config"]["workload"] == "group_limited"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    res = run_bench(["--impl", "reference", "--steps", "1", "--warmup", "0"],
                    {"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"})
    assert res.returncode == 0, res.stderr
    assert res.stdout.strip() == ""


def test_reference_arm_sample_shrinks_to_its_time_budget():
    res = run_bench(["--impl", "reference", "--steps", "20", "--warmup", "1"],
                    {"EP_BENCH_REFERENCE_BUDGET_S": "0.5"})
    assert res.returncode == 0, res.stderr
    d = json.loads(res.stdout.strip())
    assert "first 64 tokens" in d["cpu_baseline"]["sample"]
    assert d["steps"] == 20 and d["value"] > 0


def test_cpu_baseline_reports_the_all_core_run():
    """The CUDA arm's cpu_baseline: the single-threaded oracle (cores = 1)
    and, beside it, the same oracle over token shards on all host threads
    (cores = the threads it used); both on a bounded sample."""
    sys.path.insert(0, ROOT)
    import bench
    from combine_ep_layout_10_b200 import workloads as W
    w = W.WORKLOADS["prefill"].scaled(T=256)
    cb = bench.cpu_baseline(w, 0, budget_s=0.2, n_tok=64)
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] > 0
    ac = cb["all_cores"]
    assert ac["cores"] == min(os.cpu_count() or 1, 64) and ac["value"] > 0
    assert "shards" in ac["sample"] and ac["unit"] == "GB/s"
