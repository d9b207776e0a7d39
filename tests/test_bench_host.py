"""Host logic of the multi-GPU benchmark, run as two gloo ranks on CPU: every
rank gets its own input seed, the job time is the max over ranks, the
weak-scaling rate counts the voxels of all ranks, and the batched workload's
elements are split over the ranks (each element on exactly one rank, batch
indices renumbered per rank) with a strong-scaling rate."""
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
                     bench.job_rate(1000, world, job_ms / 1e3),
                     bench.sum_over_ranks(1.5 + rank, "cpu"))
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
    assert res[0][3] == res[1][3] == pytest.approx(4.0)    # a per-rank quantity summed


def test_single_process_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.sum_over_ranks(3.5, "cpu") == 3.5
    assert bench.job_rate(10, 1, 2.0) == 5.0


def _run_bench(args, env_extra=None):
    import json
    import subprocess
    import sys
    env = dict(os.environ, **(env_extra or {}))
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                       env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    return [json.loads(l) for l in lines]


def test_reference_arm_line():
    """`bench.py --impl reference` (the C++ oracle on the host cores) prints one
    JSON line with the contract's keys, the same metric and workload keys as the
    GPU arm, a cpu_baseline describing the run and an e2e with no copies."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    lines = _run_bench(["--impl", "reference", "--workload", "shell_bf16", "--steps", "2",
                        "--warmup", "1"])
    assert len(lines) == 1
    d = lines[0]
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["unit"] == "voxels/s" and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 1 and d["value"] > 0
    wl = bench._workload("shell_bf16")
    cfg = d["config"]
    for key in ("workload", "n_voxels", "cin", "cout", "grid_dim", "batch"):
        assert cfg[key] == bench._workload_config(wl, 0.0)[key], key
    assert 1.0 <= cfg["nnz_avg"] <= 27.0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_without_work():
    assert _run_bench(["--impl", "reference", "--workload", "shell_bf16", "--steps", "1",
                       "--warmup", "1"], {"RANK": "1", "WORLD_SIZE": "2"}) == []


def _four_elements():
    """Four batch elements of different sizes (the batched workload's structure:
    independent sets that share no neighbour), raster order."""
    import numpy as np
    parts = []
    for b, n in enumerate((5, 9, 3, 7)):
        rng = np.random.default_rng(b)
        cells = np.sort(rng.choice(6 ** 3, n, replace=False))
        zyx = np.stack(np.unravel_index(cells, (6, 6, 6)), 1)
        parts.append(np.concatenate([np.full((n, 1), b), zyx], 1).astype(np.int32))
    return np.concatenate(parts)


def _split_rank_main(rank, world, port, out):
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
        coords = _four_elements()
        elems = bench.batch_elements(rank, world, 4)
        sub = bench.split_batch(coords, elems)
        local_ms = 4.0 * sub.shape[0]          # time grows with the rank's rows
        job_ms = bench.max_over_ranks(local_ms, "cpu")
        out[rank] = (elems, sub.tolist(), job_ms)
    finally:
        dist.destroy_process_group()


def test_two_rank_batch_split():
    import numpy as np
    import sys
    sys.path.insert(0, ROOT)
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_split_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    coords = _four_elements()
    assert res[0][0] == [0, 2] and res[1][0] == [1, 3]     # rank r: elements r, r + world
    seen = []
    for r in range(world):
        sub = np.array(res[r][1], np.int32)
        for new_b, b in enumerate(res[r][0]):
            mine = sub[sub[:, 0] == new_b]
            orig = coords[coords[:, 0] == b]
            assert np.array_equal(mine[:, 1:], orig[:, 1:])  # same rows, same order
            seen.append(b)
        assert set(sub[:, 0].tolist()) == set(range(len(res[r][0])))  # renumbered 0..m-1
    assert sorted(seen) == [0, 1, 2, 3]                      # every element exactly once
    rows = [len(res[r][1]) for r in range(world)]
    assert sum(rows) == coords.shape[0]
    job_ms = res[0][2]
    assert job_ms == res[1][2] == 4.0 * max(rows)            # the slowest rank's time
    # strong scaling: the job's rate counts the batch's voxels once
    assert coords.shape[0] == 24
    assert coords.shape[0] / (job_ms / 1e3) == pytest.approx(24 / (4.0 * max(rows) / 1e3))


def test_batch_split_more_ranks_than_elements():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert [bench.batch_elements(r, 8, 4) for r in range(8)] == [[0], [1], [2], [3], [], [], [], []]
    assert bench.batch_elements(0, 1, 4) == [0, 1, 2, 3]
    assert bench.split_batch(_four_elements(), []).shape == (0, 4)
