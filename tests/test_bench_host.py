"""bench.py's reference arm (the fp64 oracle on the host cores) on small
workloads: it runs without a GPU and prints one JSON line with the keys the
benchmark contract asks for."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    return json.loads(lines[0])


@pytest.mark.parametrize("args", [("--workload", "tiny"),
                                  ("--loss", "kl", "--kl-workload", "soft_kl_small")])
def test_reference_arm_prints_the_contract_line(args):
    d = _run(*args, "--impl", "reference", "--steps", "1", "--warmup", "3")
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert "workload" in d["config"]


def test_warmup_below_three_is_rejected():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "2"],
                         capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert out.returncode != 0


def _bench_module():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_cpu_sample_grows_past_fixed_costs_and_stops():
    grow = _bench_module().grow_sample
    calls = []

    def fixed_plus_rows(R):  # 1.5 s per call plus 8 ms per row
        calls.append(R)
        return 1.5 + 0.008 * R
    R, t = grow(fixed_plus_rows, 2048, 15.0, 8, 8)
    # one calibration run would have taken 8 rows' 1.56 s as the per-row cost
    assert 7.5 <= t <= 15.0 and R % 8 == 0 and calls[-1] == R and calls == sorted(calls)
    # a batch smaller than the target ends at all of its rows, quantum or not
    calls.clear()
    assert grow(lambda R: calls.append(R) or 1e-3 * R, 230, 2.0, 8, 8)[0] == 230
    assert len(calls) <= 3
    assert grow(lambda R: 1e-3 * R, 5, 2.0, 8, 8)[0] == 5
