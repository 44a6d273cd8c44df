"""bench.py's output contract on CPU: the reference arm's JSON line, and the
rule that a DRAM-traffic figure from an ncu capture is reported only while
the kernel sources it was taken on are unchanged."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_traffic_record_is_dropped_once_the_sources_change(monkeypatch):
    recs = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    name, rec = next(iter(recs.items()))
    monkeypatch.setattr(bench, "source_sha", lambda *names: rec["source_sha"])
    assert bench.ncu_traffic(name) == float(rec["dram_bytes_per_launch"])
    monkeypatch.setattr(bench, "source_sha", lambda *names: "0" * 16)
    assert bench.ncu_traffic(name) is None
    assert bench.ncu_traffic("no_such_kernel") is None


def test_reference_arm_labels_a_row_slice_as_extrapolated(monkeypatch, capsys):
    """When whole oracle matvecs would not fit the run's time budget, each step
    is a row slice, value is scaled to the full matvec, ms_per_step stays the
    time a step really took, and the line says so."""
    import numpy as np
    import argparse
    monkeypatch.setattr(bench, "oracle_workload", lambda rows=bench.IN_DIM, seed=4, n_vecs=4: (None, rows, [None]))
    calls = []

    def fake_time(prep, vs, min_calls, budget_s=0.0):
        calls.append((prep, min_calls))
        return (10.0 if prep == bench.IN_DIM else 10.0 * prep / bench.IN_DIM), max(min_calls, 1), 1.0

    monkeypatch.setattr(bench, "time_oracle_calls", fake_time)
    monkeypatch.delenv("RANK", raising=False)
    bench.run_reference(argparse.Namespace(steps=2000, warmup=200, gpus=1))
    d = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    ex = d["extrapolated"]
    assert ex is not None and ex["rows_per_step"] < bench.IN_DIM
    assert np.isclose(d["value"], d["ms_per_step"] * 1e3 * ex["scale_to_full_matvec"])
    assert d["ms_per_step"] * d["steps"] / 1e3 <= bench.REFERENCE_BUDGET_S * 1.01


def test_reference_arm_prints_one_contract_line():
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "us" and d["higher_is_better"] is False
    assert d["metric"] == bench.METRIC and d["value"] > 0 and d["steps"] == 1
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "us", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith("approx GEMV W 4096x14336")


def test_byte_counts_per_path():
    """Algorithmic bytes: 3 per used product, the 16 fp16 probes of every
    row, v and out; read bytes: what the call plans to read per path (dense
    panel rows, stored chunks) plus the same probes, v and out.  At effort 1
    the read figure is the dense copy's 2 bytes per entry, so a bandwidth
    computed from it cannot exceed a copy's."""
    import bench
    I, O = 4096, 14336
    assert bench.algorithmic_bytes(I, O, 0) == 32 * I + 4 * I + 4 * O
    assert bench.algorithmic_bytes(I, O, 1000) - bench.algorithmic_bytes(I, O, 0) == 3000
    assert bench.read_bytes(I, O, 2 * I * O, 0) == 2 * I * O + 32 * I + 4 * I + 4 * O
    assert bench.read_bytes(I, O, 10, 20, v_bytes=2) == 30 + 32 * I + 2 * I + 4 * O
    assert bench.read_bytes(I, O, 2 * I * O, 0) < bench.algorithmic_bytes(I, O, I * O)


def test_q8_byte_counts():
    """Q8: 2 bytes per used product, and the row scales (2 bytes per row) on
    top of the probes, v and out; at effort 1 the planned read is the int8
    dense copy, half the fp16 one."""
    import bench
    I, O = 4096, 14336
    assert bench.algorithmic_bytes_q8(I, O, 0) == 32 * I + 2 * I + 4 * I + 4 * O
    assert bench.algorithmic_bytes_q8(I, O, 1000) - bench.algorithmic_bytes_q8(I, O, 0) == 2000
    assert bench.read_bytes_q8(I, O, I * O, 0) == I * O + 32 * I + 2 * I + 4 * I + 4 * O
    assert bench.read_bytes_q8(I, O, I * O, 0) < bench.read_bytes(I, O, 2 * I * O, 0)
