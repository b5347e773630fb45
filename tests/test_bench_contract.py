"""The JSON line of bench.py's reference arm, on CPU: the arm times the fp64
oracle on host cores, so it runs here. Checks the keys and types of the line
a caller parses (metric, value, unit, steps, config, cpu_baseline, e2e) and that
the arm's value is the oracle's FLOPs over its own time, and that ranks other
than 0 print nothing."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT,
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    return [ln for ln in r.stdout.splitlines() if ln.strip()]


def test_reference_arm_line():
    lines = _run(["--impl", "reference", "--workload", "gpt2_small", "--steps", "2",
                  "--warmup", "1"])
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["config"]["workload"].startswith("gpt2_small")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert cb["unit"] == d["unit"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0
    # value = FLOPs of the timed samples / their time: one (batch, head) unit
    # of the dense GPT-2-shaped workload is 14 * d * N^2 FLOP
    flops = 2 * 14 * 64 * 1024 * 1024
    assert abs(d["value"] - flops / (2 * d["ms_per_step"] / 1e3) / 1e12) <= 1e-9 * d["value"]


def test_reference_arm_other_ranks_are_silent():
    lines = _run(["--impl", "reference", "--workload", "gpt2_small", "--steps", "1",
                  "--warmup", "0"], {"RANK": "1", "WORLD_SIZE": "2"})
    assert lines == []


class _DoneProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def test_clock_sampler_summary(tmp_path):
    """The clocks summary from nvidia-smi samples: median SM clock, maximum of
    the max clock, the active throttle reasons decoded from the bitmask (idle
    dropped), malformed lines skipped."""
    import bench
    p = tmp_path / "clocks.csv"
    p.write_text("0, 1890, 1965, 950.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
                 "0, 1920, 1965, 990.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
                 "0, 1800, 1965, 1001.0, 0x0000000000000044, Not Active, Active, Not Active, Active\n"
                 "0, 1965, 1965, 300.0, 0x0000000000000001, Not Active, Not Active, Not Active, Not Active\n"
                 "garbage line\n"
                 "0, [N/A], 1965, 1.0, 0x0, a, b, c, d\n")
    s = bench.ClockSampler(0)
    s.proc, s.path, s.out = _DoneProc(), str(p), open(p, "a")
    got = s.stop()
    assert got["samples"] == 4
    assert got["sm_mhz"] == 1905.0 and got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]


def test_clock_sampler_without_nvidia_smi():
    import bench
    s = bench.ClockSampler(0)
    assert s.stop()["reasons"] == ["unavailable"]


def test_reference_arm_forward_only_workload():
    """The fp32 workload has no backward: the arm times the oracle forward and
    counts 4 * d * N^2 FLOP per step."""
    lines = _run(["--impl", "reference", "--workload", "fp32_n512_d32", "--steps", "2",
                  "--warmup", "0"])
    d = json.loads(lines[0])
    assert d["config"]["workload"].startswith("fp32_n512_d32") and "forward" in d["config"]["workload"]
    assert "forward+backward" not in d["cpu_baseline"]["sample"]
    flops = 2 * 4 * 32 * 512 * 512
    assert abs(d["value"] - flops / (2 * d["ms_per_step"] / 1e3) / 1e12) <= 1e-9 * d["value"]


def test_peak_choice_follows_the_timed_region():
    """The roofline compares with the burst bf16 peak for a short timed region
    and with the sustained one once the region is long enough to run under the
    power cap, or its clock record shows the cap holding the clock down; both
    fractions are always reported."""
    import bench
    peaks = {"bf16_tflops": 1669.2, "bf16_tflops_sustained": 1401.3}
    free = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    capped = {"sm_mhz": 1770.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    flag_only = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.select_bf16_peak(peaks, "measured", 50.0, free)[0] == 1669.2
    assert bench.select_bf16_peak(peaks, "measured", 50.0, flag_only)[0] == 1669.2
    assert bench.select_bf16_peak(peaks, "measured", 50.0, capped)[0] == 1401.3
    assert bench.select_bf16_peak(peaks, "measured", 500.0, free)[0] == 1401.3
    # no sustained figure: always the burst one
    assert bench.select_bf16_peak({"bf16_tflops": 1669.2}, "measured", 500.0, capped)[0] == 1669.2
    assert bench.select_bf16_peak(None, "fallback", 500.0, capped)[0] == bench.FALLBACK_PEAK_TFLOPS
    roof = bench.tensor_roofline("bwd_main", 800.0,
                                 bench.select_bf16_peak(peaks, "measured", 500.0, free), None)
    assert abs(roof["frac"] - 800.0 / 1401.3) < 1e-12
    assert abs(roof["frac_of_burst"] - 800.0 / 1669.2) < 1e-12
    assert abs(roof["frac_of_sustained"] - 800.0 / 1401.3) < 1e-12
    assert "sustained" in roof["peak_kind"]
