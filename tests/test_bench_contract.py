"""bench.py's JSON contract, checked on the reference arm (the oracle on the host cores), which
runs without a GPU. The GPU arm prints the same keys plus roofline, clocks and gpu_launches."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"],
                         cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference"
    assert d["unit"] == "GB/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["steps"] == 1 and d["warmup"] == 3
    assert d["config"]["workload"].startswith("qwen3-8b weight sync")
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_warmup_below_three_is_rejected():
    out = subprocess.run([sys.executable, "bench.py", "--steps", "1", "--warmup", "2"], cwd=ROOT,
                         capture_output=True, text=True, timeout=120)
    assert out.returncode != 0 and "--warmup" in out.stderr


def test_breakeven_fit_recovers_the_stage_cost_model():
    """t = delta + c * tokens per path (Table 7's stage cost model), m* = d_delta / d_c."""
    import pytest

    sys.path.insert(0, ROOT)
    import bench

    pts = [{"tokens": T, "bf16_ms": 0.020 + 2.0e-4 * T, "mxfp8_ms": 0.030 + 1.3e-4 * T}
           for T in bench.BREAKEVEN_TOKENS]
    f = bench.breakeven_fit(pts)
    assert f["bf16"]["delta_ms"] == pytest.approx(0.020, abs=1e-4)
    assert f["mxfp8"]["c_us_per_token"] == pytest.approx(0.13, rel=1e-3)
    assert f["m_star_tokens"] == pytest.approx(0.010 / 7.0e-5, rel=1e-3)
    # No saving per token: no break-even.
    flat = [{"tokens": T, "bf16_ms": 1.0, "mxfp8_ms": 2.0} for T in bench.BREAKEVEN_TOKENS]
    assert bench.breakeven_fit(flat)["m_star_tokens"] is None


def test_breakeven_fit_from_paired_differences():
    """With paired differences the difference line is fitted directly; on exact data it agrees with
    the two per-path fits."""
    import pytest

    sys.path.insert(0, ROOT)
    import bench

    pts = [{"tokens": T, "bf16_ms": 0.020 + 2.0e-4 * T, "mxfp8_ms": 0.030 + 1.3e-4 * T,
            "diff_ms": 0.010 - 7.0e-5 * T} for T in bench.BREAKEVEN_TOKENS]
    f = bench.breakeven_fit(pts)
    assert f["delta_delta_ms"] == pytest.approx(0.010, abs=1e-4)
    assert f["delta_c_us_per_token"] == pytest.approx(0.07, rel=1e-3)
    assert f["m_star_tokens"] == pytest.approx(0.010 / 7.0e-5, rel=1e-3)


def test_clock_window_picks_the_samples_of_a_timed_region():
    """Each secondary line reports the SM clock sampled while it was timed, or the nearest sample
    when its window is shorter than the sampling interval."""
    import bench

    cs = bench.ClockSampler(0)
    flags = "Not Active, Not Active, Not Active"
    cs.lines = [f"1965, 1965, 700, 0x0, {flags}, Not Active", f"1800, 1965, 950, 0x4, {flags}, Active",
                f"1700, 1965, 990, 0x4, {flags}, Active"]
    cs.times = [10.0, 10.1, 10.2]
    w = cs.window(10.05, 10.25)
    assert w["sm_mhz"] == 1750 and w["samples"] == 2 and w["reasons"] == ["sw_power_cap"]
    w = cs.window(9.0, 9.01)
    assert w["sm_mhz"] == 1965 and w["samples"] == 1 and w["reasons"] == []
    assert bench.ClockSampler(0).window(0.0, 1.0) == {}
