"""Host logic of the multi-GPU bench path on CPU with gloo, world size 2.

The path shards by batch sample with no collective on the data path; the only
cross-rank step is taking the slowest rank's time.  These tests run two gloo
ranks as separate processes and check that each rank draws its own batch and
that both agree on the max-over-ranks time and the whole-job throughput.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import synthetic
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        total = bench.max_over_ranks(local_ms, dist, torch.device("cpu"))
        value = bench.job_throughput(2e9, world, 4, total)
        wl = synthetic.WORKLOADS["subm_small"]
        coords = synthetic.uniform_cube(seed=bench.rank_seed(wl.seed, rank), **wl.gen_args)
        np.save(os.path.join(out_dir, f"coords{rank}.npy"), coords)
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(f"{total} {value}")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_use_distinct_batches(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    got = [tuple(map(float, open(tmp_path / f"r{r}.txt").read().split())) for r in range(world)]
    assert got[0] == got[1]
    total, value = got[0]
    assert total == 15.0
    assert value == pytest.approx(2e9 * world * 4 / 15e-3 / 1e12)
    c0, c1 = np.load(tmp_path / "coords0.npy"), np.load(tmp_path / "coords1.npy")
    assert c0.shape == c1.shape and not np.array_equal(c0, c1)
