"""Host logic of the multi-GPU benchmark, run as two gloo ranks on CPU: every
rank gets its own input seed, the job time is the max over ranks, and the
weak-scaling rate counts the voxels of all ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slowest
        job_ms = bench.max_over_ranks(local_ms, "cpu")
        out[rank] = (bench.feature_seed(rank), job_ms,
                     bench.job_rate(1000, world, job_ms / 1e3))
    finally:
        dist.destroy_process_group()


def test_two_rank_reduction_and_rate():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    seeds = {res[r][0] for r in range(world)}
    assert len(seeds) == world                        # each replica has its own input
    assert res[0][1] == res[1][1] == pytest.approx(15.0)   # max over ranks on every rank
    assert res[0][2] == pytest.approx(2 * 1000 / 0.015)    # all ranks' voxels / job time


def test_single_process_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.job_rate(10, 1, 2.0) == 5.0
