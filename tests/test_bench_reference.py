"""The reference arm of bench.py (the CPU oracle on the same workload): one JSON line with the
GPU arm's metric, unit, direction and workload keys, timed after untimed warm-up tokens."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(os.cpu_count() is None, reason="needs the host core count")
def test_reference_arm_line():
    import bench

    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")   # the CPU draw of the seeded layer, as on a box without a GPU
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2", "--warmup", "3"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["steps"] >= 1 and d["warmup"] >= 3
    wl = bench.WORKLOADS["decode"]
    cfg = d["config"]
    assert cfg["workload"] == wl["desc"]
    assert (cfg["n_tokens_per_step"], cfg["hidden"], cfg["expert_inter"], cfg["experts"], cfg["top_k"]) == \
        (wl["n"], wl["H"], wl["I"], wl["E"], wl["k"])
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] == os.cpu_count()
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
