"""The bench's reference arm (the oracle timed on the host cores) prints one JSON line with the
keys the measurement contract asks for; under torchrun only rank 0 prints. Runs on CPU."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
        "cpu_baseline", "e2e"}


def _run(env_extra=None):
    env = dict(os.environ, **(env_extra or {}))
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                          "--warmup", "0", "--cpu-sample-tokens", "2"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    return [line for line in out.stdout.splitlines() if line.strip()]


def test_reference_arm_prints_one_contract_line():
    lines = _run()
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert KEYS <= set(d)
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"]


def test_reference_arm_other_ranks_print_nothing():
    assert _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []


def test_one_core_oracle_sample_runs_with_one_blas_thread(monkeypatch):
    """The one-core CPU baseline re-times the same prepared sample with the BLAS pool held to
    one thread, and reports that as its core count."""
    sys.path.insert(0, ROOT)
    import bench
    from threadpoolctl import threadpool_info
    seen = {}

    def fake_sample(tokens, prepared=None):
        seen["tokens"], seen["prepared"] = tokens, prepared
        seen["threads"] = max((d.get("num_threads", 1) for d in threadpool_info()), default=1)
        return 4.0, 8.0, prepared

    monkeypatch.setattr(bench, "oracle_sample", fake_sample)
    one = bench.oracle_sample_one_core(32, "prepared-sample")
    assert seen == {"tokens": 32, "prepared": "prepared-sample", "threads": 1}
    assert one == {"value": 4.0, "unit": bench.UNIT, "cores": 1, "seconds": 8.0}


class _FakeNvml:
    """Stands in for pynvml: SM clock cycles 1700, 1800, 1900 MHz, 900 W, power cap active."""
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonSwPowerCap = 0x4
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonHwThermalSlowdown = 0x40

    def __init__(self, fail_init=False):
        self.fail_init, self.n, self.shut = fail_init, 0, False

    def nvmlInit(self):
        if self.fail_init:
            raise RuntimeError("no NVML")

    def nvmlShutdown(self):
        self.shut = True

    def nvmlDeviceGetHandleByIndex(self, i):
        return ("gpu", i)

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        assert kind == self.NVML_CLOCK_SM
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        assert kind == self.NVML_CLOCK_SM
        self.n += 1
        return (1700, 1800, 1900)[self.n % 3]

    def nvmlDeviceGetPowerUsage(self, h):
        return 900_000                                  # mW

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return 0x4 | 0x1                               # power cap + idle bit (not reported)


def test_clock_sampler_reads_nvml_during_the_region(monkeypatch):
    sys.path.insert(0, ROOT)
    import time
    import bench
    fake = _FakeNvml()
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    with bench.ClockSampler(0) as clk:
        time.sleep(0.1)
    s = clk.summary()
    assert fake.shut and s["source"].startswith("nvml")
    assert s["samples"] >= 5 and s["sm_mhz"] in (1700.0, 1800.0, 1900.0)
    assert s["sm_max_mhz"] == 1965.0 and s["power_w_max"] == 900.0
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_sampler_falls_back_when_nvml_is_missing(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setitem(sys.modules, "pynvml", _FakeNvml(fail_init=True))
    monkeypatch.setenv("PATH", "/nonexistent")      # and no nvidia-smi either: no record
    with bench.ClockSampler(0) as clk:
        pass
    assert clk.nvml is None and clk.summary() is None
