"""The benchmark's reference arm (`bench.py --impl reference`): the oracle
timed on the host cores, on the same workload, metric and unit as the CUDA
arm.  It needs no GPU, so it runs here: one JSON line from rank 0 with the
keys the line contract names, nothing from the other ranks.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env=None):
    env = dict(os.environ)
    env.update(extra_env or {})
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                           "--warmup", "0"], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=600)


def test_reference_arm_prints_one_line():
    r = _run()
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    import bench
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["higher_is_better"] is True and line["value"] > 0
    assert line["config"]["workload"] == "topk480"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"],
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    r = _run({"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_clock_sampler_reads_nvml_reasons(monkeypatch):
    """The timed region's clock record: a fake NVML reports a capped clock
    with the power-cap and hardware-slowdown bits set; the sampler takes
    several samples inside a 30 ms region and names both reasons."""
    import threading
    import time
    import types
    sys.path.insert(0, ROOT)
    import bench

    calls = {"n": 0}
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=1,
        nvmlDeviceGetMaxClockInfo=lambda h, k: 1965,
        nvmlDeviceGetClockInfo=lambda h, k: (calls.__setitem__("n", calls["n"] + 1), 1800)[1],
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: 0x4 | 0x8,
        nvmlShutdown=lambda: None)
    monkeypatch.setattr(bench.ClockSampler, "_nvml_handle", lambda self: (fake, object()))
    c = bench.ClockSampler(0)
    c.start()
    time.sleep(0.03)
    rec = c.stop()
    assert rec["source"] == "nvml"
    assert rec["samples"] >= 5 and rec["samples"] == calls["n"]
    assert rec["sm_mhz"] == 1800 and rec["sm_max_mhz"] == 1965
    assert rec["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert not any(t.name == c.thread.name and t.is_alive() for t in threading.enumerate())
    # A capped clock holds the attention kernel to the sustained peak.
    peak, label = bench.choose_peak({"bf16_tflops": 1636.8, "bf16_tflops_sustained": 1388.9},
                                    30.0, rec)
    assert label == "bf16 sustained" and peak == 1388.9
