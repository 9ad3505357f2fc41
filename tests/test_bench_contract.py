"""bench.py's reference arm (the oracle timed on the host cores) prints the contract's JSON line (CPU).

The GPU arm needs a B200; this checks, without a GPU, that the reference arm runs on a bounded
sample of the default workload and reports the same metric, unit, direction and config with the
fields the contract names, and the host-side rules of both arms (the trajectory bound, the
end-to-end step count and head groups).
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
    assert d["scaling"] == "strong" and d["data"] == "synthetic" and d["vs_baseline"] is None
    assert d["config"]["workload"].startswith("stress layer: B=2 H=40 N=75600")
    assert d["config"]["B"] == 2 and d["config"]["H"] == 40 and d["config"]["tau"] == [-3.0]
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


def test_runs_stay_inside_the_trajectory():
    """The default run (5 warm-up + 20 timed steps) fits the stress layer's 30 steps; a longer one
    is refused rather than extended with a made-up threshold."""
    import pytest

    import bench
    from temporal_block_sparse_b200 import workload as wl

    w = wl.WORKLOADS[bench.DEFAULT_WORKLOAD]
    assert w.steps == 30
    bench.check_trajectory(w, 25)
    bench.check_trajectory(w, 30)
    with pytest.raises(SystemExit):
        bench.check_trajectory(w, 31)
    assert bench.tau_at(w, 29, None) == -3.0
    with pytest.raises(ValueError):
        bench.tau_at(w, 30, None)
    with pytest.raises(ValueError):
        bench.tau_at(wl.WORKLOADS["480p"], 10, None)


def test_e2e_step_count():
    import bench

    gb = 1 << 30
    assert bench.e2e_step_count(None, 20, 5 * gb, 600 * gb) == bench.E2E_DEFAULT_STEPS == 5
    assert bench.e2e_step_count(None, 3, 5 * gb, 600 * gb) == 3     # never more than the timed steps
    assert bench.e2e_step_count(None, 20, 5 * gb, 60 * gb) == 4     # 20 GB for inputs -> 4 steps
    assert bench.e2e_step_count(None, 20, 5 * gb, 1 * gb) == 1      # never fewer than one
    assert bench.e2e_step_count(3, 20, 5 * gb, 1 * gb) == 3         # an explicit request wins
    assert bench.e2e_step_count(50, 20, 5 * gb, 1 * gb) == 20       # ... up to the timed steps


def test_mask_kernel_bytes():
    import torch

    import bench

    m = torch.zeros((2, 40, 591, 19), dtype=torch.int32)
    rows = 2 * 40 * 591
    assert bench.mask_bytes(m, 1000, 591, with_copy=False) == rows * 19 * 4 + 2000 + rows * 4
    assert bench.mask_bytes(m, 1000, 591, with_copy=True) == 2 * rows * 19 * 4 + 2000 + rows * 4


def test_kernel_hash_ignores_comments_only():
    """The hash that ties a stored DRAM-traffic figure to the code it was captured on survives a
    comment edit and changes with any edit to the code."""
    import bench
    code = "int f(int x) {\n  // the input, doubled\n  return 2 * x; /* twice */\n}\n"
    recommented = "/* f doubles its input */\nint f(int x) {\n  return 2 * x;   // same code\n}\n"
    changed = "int f(int x) {\n  return 3 * x;\n}\n"
    assert bench.code_text(code) == bench.code_text(recommented)
    assert bench.code_text(code) != bench.code_text(changed)
