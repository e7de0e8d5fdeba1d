"""bench.py's JSON contract, on CPU: the reference arm (the CPU oracle on a
bounded sample) prints one line with the keys the contract names, and the
helpers that the GPU arm uses behave on the host."""
from __future__ import annotations

import json
import os
import subprocess
import sys

from conftest import ROOT

KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"}


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--log2n", "16", "--steps", "2", "--warmup", "1"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert KEYS <= set(d)
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 1
    assert d["value"] > 0 and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["config"]["workload"].startswith("flat fp32 tensor")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] == d["value"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["h2d_bytes_per_step"] == 0
    assert e2e["d2h_bytes_per_step"] == 0


def test_traffic_lookup_and_clock_sampler_on_the_host():
    sys.path.insert(0, ROOT)
    import bench
    t = bench.traffic_for("k_quant_zre", 1 << 28)
    assert t is None or (isinstance(t, int) and t > 0)
    assert bench.traffic_for("no_such_kernel", 1 << 28) is None
    s = bench.ClockSampler(None)          # no GPU here: reports why, does not fail
    s.mark("start")
    s.mark("end")
    c = s.stop()
    assert "sm_mhz" in c and "reasons" in c
