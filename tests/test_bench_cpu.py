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


def test_plan_launch_count_follows_the_workspace_layout():
    """bench.py claims a score and a selection launch per strip batch of the plan; the
    batch count it computes must be the one the library's workspace layout implies
    (strips of 128 query blocks, as many per batch as the workspace holds)."""
    import importlib.util
    import math

    from free_block_sparse_mean_b200 import _lib
    from free_block_sparse_mean_b200._lib import SaShape
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    lib = _lib.load()
    al = lambda x: (x + 255) // 256 * 256
    for B, H, N, d in ((1, 24, 118800, 128), (1, 40, 75600, 128), (1, 24, 4096, 128), (2, 3, 20000, 64),
                       (1, 2, 262144, 64)):
        Nb, BH = math.ceil(N / 64), B * H
        W = (Nb + 31) // 32
        pair_in_smem = Nb <= 1207        # the pairing's bitsets fit in shared memory up to here
        fixed = (2 * al(BH * Nb * d * 4) + al(BH * Nb * 8) + al(BH * Nb * W * 4)
                 + (0 if pair_in_smem else al(BH * Nb * W * 4)))
        strip = 128 * ((Nb + 31) // 32 * 32) * 4
        per = (int(lib.sparse_attn_plan_workspace_size(SaShape(B, H, N, d, 64))) - fixed) // strip
        strips = BH * math.ceil(Nb / 128)
        assert 1 <= per <= strips
        assert bench.plan_batches(BH, Nb) == math.ceil(strips / per), (B, H, N, d)
