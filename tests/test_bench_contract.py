"""The JSON line of bench.py's reference arm (CPU oracle), as the driver reads it, and the
bench's host-side rules."""
import importlib.util
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_contract", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_reference_arm_json_line():
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    bench = _load_bench()
    wl = bench.I.WORKLOADS["prefill128k"]
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC["prefill128k"][0] and d["unit"] == "tokens/s"
    assert d["higher_is_better"] is True and d["steps"] == 3 and d["warmup"] == 3
    assert d["config"] == bench.workload_config(wl, 1)  # the same config object as the CUDA arm's
    assert d["value"] > 0 and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_traffic_only_at_the_captured_sizes():
    """roofline.traffic comes from captures of each workload at its own sizes
    on contiguous caches: a run with other sizes or a paged pool reports null."""
    import dataclasses
    bench = _load_bench()
    wl = bench.I.WORKLOADS["decode"]
    assert bench.captured_traffic(wl, False) == bench.TRAFFIC["decode"] is not None
    assert bench.captured_traffic(wl, True) is None
    assert bench.captured_traffic(dataclasses.replace(wl, num_seqs=4), False) is None
    assert bench.captured_traffic(dataclasses.replace(wl, seq_len=32768, q_start=32767), False) is None
    big = bench.I.WORKLOADS["prefill128k"]
    assert bench.captured_traffic(big, False) == bench.TRAFFIC["prefill128k"] is not None
    assert bench.captured_traffic(bench.I.WORKLOADS["prefill1m"], False) is None
