"""The multi-GPU plumbing of bench.py, run as world-size-2 gloo ranks on the
CPU: data-parallel replicas with no exchange on the data path, timed as the
maximum over ranks, whole-job throughput counted over all ranks' tokens, and
the reference arm under torchrun printing one line from rank 0 while the other
rank exits without work."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ranks_body(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist

    class Args:
        pass
    w, r, _ = bench.dist_setup(Args())
    try:
        assert (w, r) == (world, rank)
        assert dist.get_backend() == "gloo"
        bench.barrier(world)
        # each rank's own time; every rank sees the slowest
        ms = 10.0 + 5.0 * rank
        ms_max = bench.max_over_ranks(ms, world)
        assert ms_max == 10.0 + 5.0 * (world - 1)
        # all ranks' tokens over the slowest rank's time
        v = bench.whole_job_value(4096, world, 3, ms_max)
        assert abs(v - 4096 * world * 3 / (ms_max / 1e3)) < 1e-6
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_count_every_rank():
    mp.spawn(_ranks_body, args=(2, free_port()), nprocs=2, join=True)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.whole_job_value(100, 1, 2, 1000.0) == 200.0


def test_reference_arm_under_torchrun_prints_once():
    env = dict(os.environ)
    env.pop("WORLD_SIZE", None)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), "bench.py", "--impl",
           "reference", "--workload", "tiny", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["config"]["parallelism"] == "replicas x2"
