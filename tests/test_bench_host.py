"""The bench's reference arm on CPU: `bench.py --impl reference` times the
float64 oracle on the host cores and prints one JSON line of the same
contract as the CUDA arm; under a multi-rank launch only rank 0 prints and
the other ranks exit 0 without work."""
import json
import os
import subprocess
import sys

ROOT = os.path.join(os.path.dirname(__file__), "..")
CMD = [sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "1",
       "--warmup", "0", "--cpu-budget", "2"]


def _run(env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run(CMD, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_prints_one_contract_line():
    proc = _run({})
    assert proc.returncode == 0, proc.stderr[-2000:]
    lines = [l for l in proc.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["unit"] == "ms" and d["higher_is_better"] is False
    assert d["value"] > 0 and d["ms_per_step"] == d["value"]
    assert d["steps"] == 1 and d["warmup"] == 0
    assert d["config"]["workload"] == "tiny"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_do_no_work():
    proc = _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert proc.returncode == 0, proc.stderr[-2000:]
    assert proc.stdout.strip() == ""


def test_rank_problem_replicas_and_kv_head_shards():
    import argparse
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from synthetic import WORKLOADS
    w = WORKLOADS["llama_512k"]
    full, kv, local = bench.rank_problem(w, argparse.Namespace(shard="heads", seed=0), rank=1, world=4)
    assert kv == [2, 3] and full.seed == 0 and full.h_q == 32
    assert (local.h_q, local.h_kv, local.seqlen) == (8, 2, w.seqlen)
    full, kv, local = bench.rank_problem(w, argparse.Namespace(shard="replicas", seed=0), rank=1, world=4)
    assert kv is None and full is local and full.seed == 1 and full.h_q == 32
