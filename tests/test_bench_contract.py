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
