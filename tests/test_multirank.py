"""The multi-GPU path of bench.py on CPU: two `gloo` ranks (no GPU).

bench.py runs one replica per rank (its own sequences, no data-path collective)
and reports the whole job's rate from the slowest rank's device time."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out_dir):
    import bench
    import synth

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        total, value = bench.job_rate(dist, torch, times[rank], 16, world, 10, "cpu")
        wl = synth.make_workload("stack20_128k", seed=rank, N=4096)
        keys = wl.ki(0)[0, :64]
        np.save(os.path.join(out_dir, f"r{rank}.npy"), np.array([total, value]))
        np.save(os.path.join(out_dir, f"k{rank}.npy"), keys)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_job_rate_and_independent_replicas(tmp_path):
    times = [123.0, 150.5]   # per-rank device time of 10 steps, ms
    mp.start_processes(_rank_main, args=(2, _free_port(), times, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    r0, r1 = np.load(tmp_path / "r0.npy"), np.load(tmp_path / "r1.npy")
    # every rank reports the slowest rank's time and the whole-job rate
    assert r0[0] == r1[0] == pytest.approx(150.5)
    assert r0[1] == pytest.approx(16 * 2 * 10 / 0.1505)
    # the replicas draw different sequences (seed = rank)
    assert not np.array_equal(np.load(tmp_path / "k0.npy"), np.load(tmp_path / "k1.npy"))


def test_single_rank_rate_needs_no_process_group():
    import bench

    total, value = bench.job_rate(None, torch, 200.0, 16, 1, 100, "cpu")
    assert total == 200.0 and value == pytest.approx(16 * 100 / 0.2)
