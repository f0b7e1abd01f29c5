"""bench.py --gpus N without torchrun spawns N processes itself (one per GPU in
a real run) with RANK / LOCAL_RANK / WORLD_SIZE / MASTER_* set, and rank 0
alone prints the JSON line.  Checked on the CPU through the reference arm (the
oracle on the host cores), which needs no GPU: the printed line must report the
N ranks, and only one line may be printed."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_spawns_ranks_and_rank0_prints_one_line():
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(k, None)
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference",
                          "--config", "tiny_decode", "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, env=env, timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["unit"] == "query-layers/s" and line["value"] > 0
