"""bench.py's host side on the CPU: the reference arm's JSON line, the rank handling of a
multi-process launch, the workload table, the peaks and the clock-sample parsing."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

BASE_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
             "vs_baseline", "dtype", "data", "config"}


def run_bench(*args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                         env=env, timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    return res.stdout


@pytest.mark.parametrize("variant", ["auto", "backward"])
def test_reference_arm_prints_one_contract_line(variant):
    out = run_bench("--impl", "reference", "--workload", "tiny", "--variant", variant, "--steps", "2",
                    "--warmup", "1", "--ref-step-seconds", "0.2")
    lines = [l for l in out.splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert BASE_KEYS <= set(line)
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "tokens/s"
    assert line["steps"] == 2 and line["warmup"] >= 3  # warm-up is raised to at least 3
    assert line["n_gpus"] == 1 and line["higher_is_better"] is True and line["dtype"] == "f64"
    assert line["metric"] == (bench.BACKWARD_METRIC if variant == "backward" else bench.METRIC)
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["N"] == 4096 and line["config"]["tokens_per_step"] >= 1


def test_reference_arm_runs_on_rank_zero_only():
    out = run_bench("--impl", "reference", "--workload", "tiny", "--steps", "1", "--ref-step-seconds", "0.1",
                    env_extra={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert out.strip() == ""


def test_workloads_are_the_benchmark_configurations():
    W = bench.WORKLOADS
    assert W["tiny"][:5] == (4096, 128, 32, 192, 4)
    for M in (1024, 2048, 4096, 8192, 16384):
        assert W[f"sweep_M{M}"][:5] == (65536, 512, 32, M, 8)
    for r in (16, 32, 64, 128):
        assert W[f"prefill_r{r}"] == (262144, 2048, r, 4096, 8, True)  # rows at unit RMS
    assert W["many_experts"][:5] == (32768, 4096, 64, 65536, 8)
    for N in (1, 8, 64, 256):
        assert W[f"decode_N{N}"][:5] == (N, 2048, 32, 4096, 8)
    for name in W:
        assert bench.describe(name).startswith(name + ": N=")


def test_peaks_measured_or_fallback(tmp_path, monkeypatch):
    hbm, tc, tc_sus, src = bench.peaks()
    assert hbm > 0 and tc > 0 and src in ("measured", "fallback")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))  # no peaks file there
    assert bench.peaks() == (6650.0, 1590.0, 1400.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 7000, "bf16_tflops": 1600}))
    assert bench.peaks() == (7000.0, 1600.0, None, "measured")


def test_clock_samples_are_summarised():
    s = bench.ClockSampler(0)

    class Done:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

        def join(self, timeout=None):
            pass

    s.proc, s.thread = Done(), Done()
    s.lines = [
        "0, 1800, 1965, 900.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1900, 1965, 950.2, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1700, 1965, 980.0, 0x0000000000000008, Active, Not Active, Not Active, Not Active",
        "garbled",
    ]
    out = s.stop()
    assert out == {"sm_mhz": 1800.0, "sm_max_mhz": 1965.0, "reasons": ["hw_slowdown", "sw_power_cap"], "samples": 3}
    assert bench.ClockSampler(0).stop() is None  # never started: no record
