"""bench.py's own arm on a B200: one JSON line with the keys and
consistency the measurement contract asks for (short runs; the numbers
themselves are not judged here)."""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def _common(d, steps, warmup, unit, bound):
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "e2e", "gpu_launches"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == steps and d["warmup"] == warmup
    assert d["unit"] == unit and d["value"] > 0 and d["higher_is_better"] is True
    assert d["dtype"] == "bf16" and d["config"]["workload"]
    r = d["roofline"]
    assert r["bound"] == bound and r["unit"] == unit and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3
    assert 0.05 < r["frac"] < 1.3
    lo, hi = r["isolated_launch_ms_p10_p90"]
    assert 0 < lo <= r["isolated_launch_ms"] <= hi
    e = d["e2e"]
    assert e["unit"] == unit and 0 < e["value"] < d["value"]
    assert e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] == steps * r["launches_per_step"]


def test_decode_bench_line():
    d = _bench("--steps", "200", "--warmup", "3", "--no-clocks", "--no-cpu-baseline",
               "--e2e-steps", "2")
    _common(d, 200, 3, "GB/s", "hbm")
    assert d["roofline"]["algorithmic_bytes_per_launch"] == d["config"]["kv_bytes_per_step"]
    import workloads
    assert d["config"]["seed"] == workloads.CONFIGS["llama70b"].seed
    pm = d["partial_merge"]
    assert pm["us_per_call"] > 0 and pm["steps"] == 200
    # the same K steps as direct calls: the graph replay removes host launch
    # work only, so the two agree closely
    dc = d["direct_calls"]
    assert 0.5 < dc["ms_per_step"] / d["ms_per_step"] < 2.0
    # the decode-loop form: only q and the new token move per step
    lp = d["e2e_decode_loop"]
    assert 0 < lp["value"] <= 1.2 * d["value"] and lp["h2d_bytes_per_step"] < 1 << 20
    # every other workload, timed the same way
    assert sorted(d["per_config"]) == sorted(n for n in workloads.CONFIGS if n != "llama70b")
    for name, e in d["per_config"].items():
        assert e["steps"] == 200 and e["warmup"] == 3 and e["us_per_call"] > 0
        assert abs(e["value_gbs"] - e["kv_bytes_per_step"] / (e["us_per_call"] * 1e3)) < 0.01 * e["value_gbs"]
        assert 0 < e["frac_of_hbm_peak"] < 1.3


def test_prefill_bench_line():
    d = _bench("--config", "llama70b_prefill2k", "--steps", "100", "--warmup", "3", "--no-clocks",
               "--no-cpu-baseline", "--e2e-steps", "2")
    _common(d, 100, 3, "TFLOP/s", "tensor")
    assert d["roofline"]["algorithmic_flops_per_launch"] == d["config"]["flops_per_step"]
