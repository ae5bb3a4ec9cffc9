"""Host-side logic of bench.py that needs no GPU: the multi-rank timing
aggregation (gloo, world size 2) and the reference arm's rank behaviour."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r took (r + 1) * 10 ms: the job is timed by the slowest rank
        t = bench.max_over_ranks(10.0 * (rank + 1), world, "cpu")
        out[rank] = (t, bench.replica_throughput(world, 1000, 5, t))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    port = 29500 + (os.getpid() % 1000)
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 20.0
    # 2 replicas x 1000 tokens x 5 steps in 20 ms
    assert res[0][1] == pytest.approx(2 * 1000 * 5 / 0.020)


def test_replica_throughput_single():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.replica_throughput(1, 16384, 10, 100.0) == pytest.approx(16384 * 10 / 0.1)


def _run_reference(rank, world):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--workload", "tiny", "--steps", "2", "--warmup", "1"],
                          capture_output=True, text=True, env=env, timeout=600)


def test_reference_arm_rank0_prints_one_json_line():
    r = _run_reference(0, 2)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["n_gpus"] == 2 and d["steps"] == 2 and d["warmup"] == 1


def test_reference_arm_other_ranks_exit_silently():
    r = _run_reference(1, 2)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_l2_flush_rule_follows_the_layer_footprint():
    """Layers touching less than twice the L2 per step are timed with an L2
    flush between steps, and their config says so; the Mixtral-shaped layer
    (weights alone 2.8 GB) is not."""
    import moe_workloads as mw
    W = mw.WORKLOADS
    # weights 3 * d * F * 2 bytes are part of the footprint
    m = W["mixtral"]
    assert bench.layer_footprint(m) > 3 * m.d_model * 8 * 14336 * 2
    assert not bench.flushes_l2(m)
    assert bench.flushes_l2(W["tiny"]) and bench.flushes_l2(W["variable_size"])
    assert not bench.flushes_l2(W["fine_grained"])
    assert "flushed" in bench.workload_config(W["tiny"], 1)["l2"]
    assert "no flush" in bench.workload_config(m, 1)["l2"]
