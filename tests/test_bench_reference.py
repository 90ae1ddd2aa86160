"""The benchmark's reference arm (the CPU oracle on the host cores) runs
without a GPU: its one JSON line must carry the keys the benchmark contract
names, with values of the right kinds."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in d, key
    assert d["value"] > 0 and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] >= 3 and d["n_gpus"] == 1
    assert "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_peak_follows_the_clocks_seen_while_timing():
    # The burst bf16 peak applies to a run at full clock; the sustained one only
    # when the timed steps ran under the power cap or well below max clock.
    import bench
    pk = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    full = {"samples": 20, "sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reason_samples": {}}
    capped = {"samples": 20, "sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reason_samples": {"sw_power_cap": 8}}
    slow = {"samples": 20, "sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "reason_samples": {}}
    none = {"samples": 0, "sm_mhz": None, "sm_max_mhz": None}
    assert bench.choose_bf16_peak(pk, full)[:2] == (1600.0, "bf16_tflops")
    assert bench.choose_bf16_peak(pk, capped)[:2] == (1400.0, "bf16_tflops_sustained")
    assert bench.choose_bf16_peak(pk, slow)[:2] == (1400.0, "bf16_tflops_sustained")
    # no samples: the stricter (larger) burst peak
    assert bench.choose_bf16_peak(pk, none)[:2] == (1600.0, "bf16_tflops")
    # a stray capped sample in a full-clock run does not switch the peak
    stray = dict(full, reason_samples={"sw_power_cap": 1})
    assert bench.choose_bf16_peak(pk, stray)[:2] == (1600.0, "bf16_tflops")
