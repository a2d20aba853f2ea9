"""bench.py's JSON line on a GPU: every key of the benchmark contract is there
and consistent with the others (a short run on a 1024-token prefix of the
headline batch, with the e2e leg and a small CPU-baseline sample)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                         capture_output=True, text=True, timeout=900, env=env, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-3000:]
    lines = [json.loads(x) for x in res.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, res.stdout
    return lines[0]


def test_bench_line_contract():
    d = _run("--tokens", "1024", "--steps", "3", "--warmup", "3", "--cpu-tokens", "16",
             "--no-skip")
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "roofline", "cpu_baseline", "e2e", "gpu_launches", "clocks"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == 3 and d["warmup"] == 3
    assert d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["dtype"] == "bf16" and d["scaling"] == "weak" and d["vs_baseline"] is None
    N = d["config"]["N"]
    assert N == 1024
    assert abs(d["value"] - N / (d["ms_per_step"] / 1e3)) <= 1e-6 * d["value"]
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert 0.0 < r["frac"] < 1.5
    assert r["traffic"] is None          # a prefix run: the committed summaries are full-size
    assert "burst" in r["peak_rule"]     # well under 2 s of timed region
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0
    e = d["e2e"]
    assert e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > e["h2d_bytes_per_step"] // 2
    assert e["value"] > 0
    assert d["gpu_launches"] >= 7 * d["steps"]     # count, two sweeps, merge, dH, dW, finish (+ split sum)
    assert d["clocks"] is None or "sm_mhz" in d["clocks"]


def test_reference_arm_line():
    d = _run("--impl", "reference", "--steps", "1", "--warmup", "3", "--ref-tokens", "8",
             "--workload", "mid")
    assert d["impl"] == "reference" and d["n_gpus"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["value"] == d["value"]
    assert set(d["config"]) == {"workload", "N", "D", "V", "parallelism", "l2"}
