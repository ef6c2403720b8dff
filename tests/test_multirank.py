"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

The path does not shard: N GPUs run N independent replicas.  What N > 1
adds is host logic -- a barrier, the max over ranks of each timed quantity,
the whole-job throughput, and rank 0 alone printing -- which these tests run
with two CPU processes.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch
    import bench
    ranks = bench.Ranks("gloo", torch.device("cpu"))
    assert (ranks.rank, ranks.world) == (rank, world)
    ranks.barrier()
    # Each rank "measured" a different step time; every rank must get the max.
    ms = ranks.max(2.0 + rank * 0.5)
    value = bench.job_throughput(1e9, ranks.world, ms)
    ranks.barrier()
    ranks.close()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"ms": ms, "value": value}, f)


def test_max_over_ranks_and_job_throughput(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for g in got:
        assert g["ms"] == 2.5                        # the slowest rank
        assert g["value"] == pytest.approx(1e9 * 2 / 2.5e-3 / 1e9)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import torch
    import bench
    env = {k: os.environ.pop(k) for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK") if k in os.environ}
    try:
        ranks = bench.Ranks("gloo", torch.device("cpu"))
        assert ranks.world == 1 and ranks.pg is None
        assert ranks.max(3.25) == 3.25
        ranks.barrier()
        ranks.close()
    finally:
        os.environ.update(env)


def test_reference_arm_under_torchrun_prints_once():
    """`bench.py --impl reference` launched as two ranks: rank 0 times the
    oracle and prints one JSON line, the other rank exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--config", "1", "--steps", "1", "--warmup", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
