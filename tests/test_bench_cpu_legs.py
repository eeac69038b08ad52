"""The benchmark's CPU legs (the oracle baselines and the reference arm) on
small workloads: they run, report what the JSON line needs, and time only the
decode work."""
import io
import json
import os
import sys
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _small():
    import residual_bit_kv_b200.synth as synth
    return synth.WORKLOADS["ouro_layer"].replace(batch=2, heads=2, tokens=128)


def test_cpu_baseline_single_core(monkeypatch):
    import bench
    monkeypatch.setattr(bench, "CPU_SAMPLE_SECONDS", 0.01)
    w = _small()
    r = bench.cpu_baseline(w)
    assert r["kind"] == "oracle" and r["cores"] == 1 and r["unit"] == "tokens/s"
    assert r["value"] > 0
    assert "decode units of layer 0" in r["sample"]


def test_cpu_baseline_all_cores(monkeypatch):
    import bench
    monkeypatch.setattr(bench, "CPU_POOL_MAX_WORKERS", 2)
    import residual_bit_kv_b200.synth as synth
    w = synth.WORKLOADS["tiny"]
    r = bench.cpu_baseline_all_cores(w)
    assert r["kind"] == "oracle" and 1 <= r["cores"] <= 2 and r["nproc"] >= 1
    assert r["value"] > 0 and r["ms_per_call"] > 0
    assert f"{r['cores'] * w.loops} (batch,head,loop)" in r["sample"]


def test_reference_arm_prints_one_line():
    import argparse
    import bench
    args = argparse.Namespace(gpus=1, steps=1, warmup=0, impl="reference")
    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.run_reference(args, rank=0) == 0
    lines = [ln for ln in buf.getvalue().splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
