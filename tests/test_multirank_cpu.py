"""The multi-GPU path is replicas: each rank runs its own copy of the workload
and the only cross-rank traffic is a barrier and a MAX of the timed span.
This exercises that host logic with two gloo ranks on the CPU."""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_path):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    elapsed = 0.5 + rank  # rank 1 is the slow replica
    mx = bench._max_over_ranks(elapsed, world, device="cpu")
    value = bench.whole_job_tokens_per_s(world, 131072, 10, mx)
    dist.barrier()
    with open("%s.%d" % (out_path, rank), "w") as f:
        f.write("%r %r" % (mx, value))
    dist.destroy_process_group()


def test_two_rank_max_and_weak_scaling(tmp_path):
    port = _free_port()
    out = str(tmp_path / "r")
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(2):
        mx, value = map(float, open("%s.%d" % (out, r)).read().split())
        assert mx == 1.5  # the slowest rank's span, seen by every rank
        assert value == pytest.approx(2 * 131072 * 10 / 1.5)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench._max_over_ranks(0.25, 1) == 0.25
    assert bench.whole_job_tokens_per_s(1, 1000, 4, 2.0) == 2000.0
