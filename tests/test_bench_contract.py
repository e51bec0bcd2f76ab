"""The reference arm of bench.py on the CPU: the oracle timed on a bounded
sample, one JSON line from rank 0 only, with the keys the line carries."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CMD = [sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "1",
       "--workload", "flat-1M-W4"]


def _run(env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run(CMD, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_prints_one_line_with_the_contract_keys():
    r = _run({"RANK": "0", "WORLD_SIZE": "1"})
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["steps"] == 1 and d["warmup"] == 1 and d["higher_is_better"] is True
    assert d["value"] > 0 and d["config"]["workload"].startswith("flat-1M-W4")
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


FAKE_SMI = """#!/usr/bin/env python3
import datetime, sys, time
while True:
    ts = datetime.datetime.now().strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    clk = 1500 if time.time() < float(sys.argv[-1]) else 1965
    print(f"{ts}, 0, {clk}, 1965, 700.00, 0x4, Not Active, Not Active, Not Active, Active", flush=True)
    time.sleep(0.02)
"""


def test_clock_sampler_reports_only_the_timed_region(tmp_path, monkeypatch):
    """The sampler waits for nvidia-smi's first sample, then keeps only the
    samples stamped between mark() and stop() (a fake nvidia-smi reports
    1500 MHz before a switch time and 1965 MHz after it)."""
    import importlib.util
    import time

    switch = time.time() + 0.6
    fake = tmp_path / "nvidia-smi"
    fake.write_text(FAKE_SMI.replace("sys.argv[-1]", repr(str(switch))))
    fake.chmod(0o755)
    monkeypatch.setenv("PATH", str(tmp_path) + os.pathsep + os.environ["PATH"])
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)

    s = bench.ClockSampler(interval_ms=20)
    s.start()
    time.sleep(max(0.0, switch - time.time()) + 0.1)
    s.mark()
    time.sleep(0.4)
    c = s.stop()
    assert c["samples"] >= 5 and c["sm_mhz"] == 1965.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]

    s = bench.ClockSampler(interval_ms=20)       # a region shorter than one interval
    s.start()
    s.mark()
    c = s.stop()
    assert c["samples"] >= 1


def test_reference_arm_other_ranks_exit_without_work():
    r = _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr
    assert not [ln for ln in r.stdout.splitlines() if ln.startswith("{")]


import pytest  # noqa: E402


def _b200_line(args):
    r = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True, text=True,
                       timeout=600, env=dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0"))
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    return json.loads(lines[0])


@pytest.mark.gpu
def test_b200_arm_small_case_prints_the_contract_keys():
    d = _b200_line(["--n", "1048576", "--workers", "4", "--steps", "5", "--warmup", "3",
                    "--adam-steps", "2", "--no-cpu-baseline", "--e2e-steps", "1"])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "roofline",
                "e2e", "gpu_launches", "clocks"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["value"] > 0 and d["gpu_launches"] == 5 * 5
    assert d["roofline"]["kernel"] == "ob_pack_kernel" and d["roofline"]["frac"] > 0
    assert d["e2e"]["value"] > 0 and d["e2e"]["h2d_bytes_per_step"] == 4 * 1048576 * 4


@pytest.mark.gpu
def test_b200_arm_split_step_mode_on_one_gpu():
    """--multi split runs the split step's calls through the bench's
    multi-GPU path (with one process there is no exchange)."""
    d = _b200_line(["--n", "1048576", "--workers", "4", "--steps", "5", "--warmup", "3",
                    "--adam-steps", "2", "--multi", "split", "--e2e-steps", "1"])
    assert d["scaling"] == "strong" and d["value"] > 0 and d["gpu_launches"] == 5 * 5
    assert "split step" in d["config"]["parallelism"]
    assert d["e2e"]["value"] > 0
