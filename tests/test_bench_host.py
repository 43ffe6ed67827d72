"""Host-side parts of bench.py, on CPU: the roofline record, the traffic records
tied to kernel sources, the clock summary, and the reference arm's JSON line."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_roofline_record():
    r = bench.roofline(13_856_391_424, 2.9e-3, traffic=14.5e9)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(13.856391424 / 2.9e-3, rel=1e-9)
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], rel=1e-12)
    assert r["frac_nominal"] == pytest.approx(r["achieved"] / 8000.0, rel=1e-12)
    assert r["peak_kind"] in ("measured", "fallback") and r["traffic"] == 14.5e9


def test_traffic_record_follows_its_kernel_sources(monkeypatch):
    # the committed records were taken on the committed kernel sources
    for w in ("rollout", "stress"):
        with open(os.path.join(ROOT, "profiles", f"scan_{w}_traffic.json")) as f:
            rec = json.load(f)
        assert rec["source_sha256"] == bench.kernel_source_hash(w), (
            f"{w}: kernel sources changed since the DRAM traffic was captured")
        assert bench.recorded_traffic(w) == rec["dram_bytes_per_launch"]
    # a source change makes the record stale: no traffic is reported
    monkeypatch.setattr(bench, "kernel_source_hash", lambda w: "0" * 64)
    assert bench.recorded_traffic("rollout") is None
    assert bench.recorded_traffic("conv") is None


def test_clock_summary_flags_throttle_reasons():
    cs = bench.ClockSampler(0)
    cs.proc = object()                      # as if nvidia-smi had run
    cs.lines = ["0, 1965, 1965, 420.5, 0x0, Not Active, Not Active, Not Active, Not Active\n",
                "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active\n",
                "0, 1785, 1965, 1001.2, 0x4, Not Active, Not Active, Not Active, Active\n",
                "0, 120, 1965, 150.0, 0x0, Not Active, Not Active, Not Active, Not Active\n"]
    s = cs.summary()
    assert s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    assert s["sm_mhz"] == 1800.0            # median over the loaded samples only


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "1"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 2
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
