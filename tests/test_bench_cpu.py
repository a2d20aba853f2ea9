"""Host logic of bench.py that needs no GPU: the clock-sample summary keeps
only the samples stamped inside the timed window, and the roofline traffic
lookup refuses counters taken on other sources."""
import datetime

import bench


class _Proc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _row(t, mhz, power, cap):
    ts = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    return [ts, "0", str(mhz), "1965", str(power), "0x4" if cap else "0x0",
            "Not Active", "Not Active", "Not Active", "Active" if cap else "Not Active"]


def _sampler(rows):
    s = bench.ClockSampler(0)
    s.proc = _Proc()
    s.rows = rows
    return s


def test_clock_summary_keeps_the_timed_window():
    t0 = 1_800_000_000.0
    rows = [_row(t0 - 0.2, 1965, 120, False), _row(t0 - 0.1, 1965, 130, False),
            _row(t0 + 0.05, 1500, 990, True), _row(t0 + 0.10, 1410, 1000, True),
            _row(t0 + 0.15, 1455, 995, True), _row(t0 + 0.5, 1965, 140, False)]
    c = _sampler(rows).stop(t0, t0 + 0.2)
    assert c["window"] == "timed region" and c["samples"] == 3
    assert c["sm_mhz"] == 1455 and c["power_w"] == 995
    assert c["sm_max_mhz"] == 1965 and c["reasons"] == ["sw_power_cap"]


def test_clock_summary_falls_back_to_all_samples():
    t0 = 1_800_000_000.0
    rows = [_row(t0 - 1.0, 1965, 120, False), _row(t0 + 1.0, 1900, 300, False)]
    c = _sampler(rows).stop(t0, t0 + 0.01)
    assert c["window"] == "whole sampler run" and c["samples"] == 2
    assert c["reasons"] == []


def test_traffic_needs_counters_of_the_current_sources():
    # a kernel with no committed summary has no traffic figure
    assert bench.traffic_for("no_such_kernel", "headline") is None


def test_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    csrc = tmp_path / "linear_diffusion_cross_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("int v = 1;\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.source_hash()
    (tmp_path / "profiles" / "ncu_k_w.txt").write_text(
        f"source_sha256: {h}\ndram_bytes_per_launch: 1.5e9\n")
    assert bench.traffic_for("k", "w") == 1.5e9
    (csrc / "k.cu").write_text("int v = 2;\n")     # the kernel changed since the capture
    assert bench.traffic_for("k", "w") is None


def test_comment_edits_keep_the_source_hash(tmp_path, monkeypatch):
    csrc = tmp_path / "linear_diffusion_cross_b200" / "csrc"
    csrc.mkdir(parents=True)
    f = csrc / "k.cuh"
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    f.write_text('// v1\nint a = 1; /* x */ const char* s = "// kept";\n')
    h1 = bench.source_hash()
    f.write_text('// v2, reworded\n\nint a = 1;   /* y */ const char* s = "// kept";\n')
    assert bench.source_hash() == h1
    f.write_text('int a = 2; const char* s = "// kept";\n')
    assert bench.source_hash() != h1
    f.write_text('int a = 1; const char* s = "// changed";\n')
    assert bench.source_hash() != h1


def _env_without_launcher():
    import os
    env = dict(os.environ)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "LOCAL_WORLD_SIZE", "MASTER_ADDR",
              "MASTER_PORT", "GROUP_RANK", "ROLE_RANK", "TORCHELASTIC_RUN_ID"):
        env.pop(k, None)
    env["OMP_NUM_THREADS"] = "1"
    return env


def test_gpus_flag_launches_that_many_ranks():
    """`bench.py --gpus 2` with no external launcher starts two ranks through
    torch.distributed.run; rank 0 prints the one JSON line with n_gpus 2 (the
    reference arm, which needs no GPU: rank 0 times the oracle, rank 1 exits
    without work)."""
    import json
    import subprocess
    import sys
    cmd = [sys.executable, bench.__file__, "--gpus", "2", "--impl", "reference",
           "--workload", "tiny", "--steps", "1", "--warmup", "3", "--ref-tokens", "8"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=600,
                         env=_env_without_launcher())
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [json.loads(x) for x in res.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = lines[0]
    assert line["n_gpus"] == 2 and line["impl"] == "reference"
    assert line["config"]["parallelism"] == "dp2"
    assert line["steps"] == 1 and line["warmup"] == 3


def test_gpus_flag_must_match_an_external_launcher(monkeypatch):
    import pytest
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    assert bench.world_from_env(2) == (2, 1, 1)
    with pytest.raises(SystemExit):
        bench.world_from_env(4)
    monkeypatch.delenv("WORLD_SIZE")
    assert bench.world_from_env(1)[0] == 1


def test_both_arms_name_the_same_config():
    from linear_diffusion_cross_b200 import synth
    for name, r in synth.RECIPES.items():
        c1 = bench.run_config(name, r, 1)
        assert c1 == bench.run_config(name, r, 1)
        assert set(c1) == {"workload", "N", "D", "V", "parallelism", "l2"}
    assert "no flush" in bench.run_config("headline", synth.RECIPES["headline"], 1)["l2"]
