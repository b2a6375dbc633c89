"""bench.py's reference arm and JSON line on the CPU: the reference arm times
the oracle on a bounded sample and prints one line with the same metric,
unit and workload as the GPU arm, an `impl` of "reference", a cpu_baseline
that describes the run and an e2e entry with no host-device traffic; under
several ranks only rank 0 works; fewer than 3 warm-up steps are raised to 3."""
import argparse
import importlib.util
import json
import os
import sys
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_contract_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_reference_line_keys(bench, monkeypatch):
    calls = []

    def fake_sample(seconds=12.0):
        calls.append(seconds)
        return 0.05 + 0.01 * len(calls), "a bounded sample", 8

    monkeypatch.setattr(bench, "oracle_sample", fake_sample)
    line = bench.run_reference(argparse.Namespace(steps=2, warmup=3), 0, 1)
    assert len(calls) == 5                                   # warm-up samples run, then the timed ones
    assert line["value"] == pytest.approx((0.09 + 0.10) / 2)  # mean of the two timed samples only
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["impl"] == "reference" and line["higher_is_better"] is True
    assert line["steps"] == 2 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["config"] == bench.bench_config(1)
    assert "workload" in line["config"] and "model" not in line["config"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["unit"] == bench.UNIT
    assert cb["cores"] == 8 and cb["sample"] == "a bounded sample"
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == bench.UNIT
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    json.dumps(line)                                          # one JSON line


def test_reference_arm_runs_on_rank_zero_only(bench, monkeypatch):
    monkeypatch.setattr(bench, "oracle_sample", lambda seconds=12.0: pytest.fail("rank 1 must not work"))
    assert bench.run_reference(argparse.Namespace(steps=1, warmup=3), 1, 2) is None


def test_warmup_is_raised_to_three(bench, monkeypatch, capsys):
    seen = {}

    def fake_reference(a, rank, world):
        seen["warmup"] = a.warmup
        return {"impl": "reference"}

    monkeypatch.setattr(bench, "run_reference", fake_reference)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--warmup", "1", "--steps", "1"])
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.delenv("RANK", raising=False)
    bench.main()
    assert seen["warmup"] == 3
    assert json.loads(capsys.readouterr().out.strip().splitlines()[-1]) == {"impl": "reference"}


def test_oracle_sample_is_bounded(bench):
    """The real sample: two 7B-shaped layers of the oracle on the host, a
    positive rate, the thread count it used, and a description."""
    t0 = time.perf_counter()
    tok_s, sample, cores = bench.oracle_sample(seconds=0.1)
    assert time.perf_counter() - t0 < 120
    assert tok_s > 0 and cores >= 1
    assert "extrapolated to 32 layers" in sample
