"""bench.py's reference arm (the oracle timed on the host cores) prints the contract's JSON line (CPU).

The GPU arm needs a B200 and is exercised by the full test run; this checks, without a GPU, that the
reference arm runs on a bounded sample and reports the same metric, unit and direction with the
fields the contract names.
"""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0", "--cpu-sample-tiles", "2"], capture_output=True, text=True, timeout=600,
                         cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    import bench
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 0
    assert d["scaling"] == "weak" and d["data"] == "synthetic" and d["vs_baseline"] is None
    assert d["config"]["workload"].startswith("480p")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_e2e_head_groups():
    """The end-to-end pipeline's head-group count: a divisor of H, fewest rounds of pair items
    over the persistent grid per step, then the most groups."""
    import bench

    # 480p: 40 heads x 128 pairs over 148 CTAs. One call takes 35 rounds, 4 groups 4 x 9 = 36,
    # 5 groups 5 x 7 = 35: five groups of eight heads.
    assert bench.e2e_head_groups(1, 40, 256, 148) == 5
    # 720p: 296 pairs a head; 8 groups of five heads take 8 x 10 = 80 rounds, as one call does
    assert bench.e2e_head_groups(1, 40, 591, 148) == 8
    # few items: never split a call that fits in one round
    assert bench.e2e_head_groups(1, 1, 16, 148) == 1
    assert bench.e2e_head_groups(1, 8, 256, 148) == 1
    for H in (1, 3, 7, 12, 40):
        assert H % bench.e2e_head_groups(1, H, 100, 148) == 0
