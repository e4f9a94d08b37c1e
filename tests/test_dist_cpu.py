"""Multi-rank host logic of bench.py on CPU: two gloo ranks.

Ranks verify disjoint request shards (no collective on the data path); the
timed region is closed by a barrier and the time is the max over ranks.
"""
import os
import socket
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CHILD = textwrap.dedent("""
    import os, sys
    sys.path.insert(0, {root!r})
    import bench
    rank, world, local = bench.dist_setup(2)
    assert world == 2 and rank == int(os.environ["RANK"])
    import torch
    mine = 10.0 + 5.0 * rank            # this rank's device time (ms)
    m = bench.max_over_ranks(mine, world, torch.device("cpu"))
    assert m == 15.0, m
    bench.barrier(world)
    seeds = bench.shard_seeds(rank)
    other = bench.shard_seeds(1 - rank)
    assert not set(seeds) & set(other)
    rate = bench.whole_job_rate(576, 10, world, m)
    assert abs(rate - 576 * 10 * 2 / 0.015) < 1e-6
    import torch.distributed as dist
    dist.destroy_process_group()
    print("rank", rank, "ok")
""")


@pytest.mark.timeout(180)
def test_two_gloo_ranks():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", CHILD.format(root=ROOT)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True))
    outs = []
    for pr in procs:
        try:
            out, _ = pr.communicate(timeout=150)
        except subprocess.TimeoutExpired:
            pr.kill()
            out, _ = pr.communicate()
        outs.append(out)
    for rank, (pr, out) in enumerate(zip(procs, outs)):
        assert pr.returncode == 0, out
        assert f"rank {rank} ok" in out


def test_whole_job_rate_single():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.whole_job_rate(576, 50, 1, 10.0) == pytest.approx(576 * 50 / 0.010)
    assert bench.shard_seeds(0) == [0, 1] and bench.shard_seeds(3) == [3000, 3001]
