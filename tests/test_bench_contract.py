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
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))["k_mac"]
    monkeypatch.setattr(bench, "source_sha", lambda *names: rec["source_sha"])
    assert bench.ncu_traffic("k_mac") == float(rec["dram_bytes_per_launch"])
    monkeypatch.setattr(bench, "source_sha", lambda *names: "0" * 16)
    assert bench.ncu_traffic("k_mac") is None
    assert bench.ncu_traffic("no_such_kernel") is None


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
