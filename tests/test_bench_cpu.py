"""The benchmark's reference arm (the CPU oracle) for the recall filter and the
clustered order: one JSON line whose config names the variant (no GPU)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("extra,key,value", [(["--recall", "0.95"], "pv_filter", "recall"),
                                             (["--cluster-iters", "1"], "cluster_iters", 1)])
def test_reference_arm_variants(extra, key, value):
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3",
           "--cpu-seconds", "0.3", *extra]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["value"] > 0 and line["config"][key] == value
    assert line["cpu_baseline"]["kind"] == "oracle"
