"""The multi-rank path of bench.py on CPU: two gloo ranks (one process each).

Each rank must run its own batch (no (b, h) problem shared, no collective on
the data path), the job time must be the slowest rank's, and the job
throughput must count every rank's work."""

import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, outdir):
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    from io_aware_exact_20_b200.workloads import WORKLOADS, make_inputs

    w = bench.rank_workload(WORKLOADS["tiny"], rank)
    q = make_inputs(w)["q"].float().numpy()
    local_ms = 10.0 + 5.0 * rank
    total = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
    np.savez(os.path.join(outdir, f"r{rank}.npz"), q=q, total=total, seed=w.data_seed)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_the_batch_and_take_the_slowest_time(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    r0, r1 = (np.load(tmp_path / f"r{r}.npz") for r in range(world))
    assert int(r0["seed"]) != int(r1["seed"])
    assert not np.array_equal(r0["q"], r1["q"])          # different data per rank
    assert float(r0["total"]) == float(r1["total"]) == 15.0  # the slowest rank


def test_job_throughput_counts_all_ranks():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.job_throughput(1, 1e12, 10, 1000.0)
    assert one == pytest.approx(10.0)
    assert bench.job_throughput(4, 1e12, 10, 1000.0) == pytest.approx(40.0)
    assert bench.max_over_ranks(3.5, 1, None) == 3.5
