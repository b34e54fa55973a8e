"""Data-parallel host path with two ranks on CPU (gloo).

The forward has no exchange between problems: each rank runs its own problem
of the workload's shape and the only collectives are the two reductions of the
timing result (max of the timed-region duration, sum of the executed FLOPs).
These tests run that host logic with world size 2 over gloo.
"""
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


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from block_sparse_linear_pool_b200 import inputs as I

        # each rank's timing result; rank 1 is the slow one
        ms = 10.0 + 5.0 * rank
        flops = 1.0e12 * (rank + 1)
        ms_max, fl_sum = bench.reduce_over_ranks(ms, flops, torch.device("cpu"))

        # each rank draws its own problem; gather a fingerprint of it
        data, cfg = I.make_workload("tiny_sla", problem=rank)
        fp = torch.tensor([float(data["Q"].float().sum()), float(data["K"].float().sum()),
                           float(data["V"].float().sum())], dtype=torch.float64)
        fps = [torch.zeros_like(fp) for _ in range(world)]
        dist.all_gather(fps, fp)
        out[rank] = (ms_max, fl_sum, [f.tolist() for f in fps], tuple(data["Q"].shape))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def _run(world):
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    return dict(out)


@pytest.fixture(scope="module")
def two_ranks():
    return _run(2)


def test_reduction_is_max_time_and_total_flops(two_ranks):
    for rank in range(2):
        ms_max, fl_sum, _, _ = two_ranks[rank]
        assert ms_max == 15.0          # the slowest rank sets the job time
        assert fl_sum == 3.0e12        # every rank's problem counts


def test_ranks_get_distinct_problems_of_one_shape(two_ranks):
    (_, _, fps0, shape0), (_, _, fps1, shape1) = two_ranks[0], two_ranks[1]
    assert shape0 == shape1
    assert fps0 == fps1                # both ranks gathered the same list
    assert not np.allclose(fps0[0], fps0[1])


def test_problem_zero_is_the_default_instance():
    from block_sparse_linear_pool_b200 import inputs as I

    a, _ = I.make_workload("tiny_sla")
    b, _ = I.make_workload("tiny_sla", problem=0)
    for k in ("Q", "K", "V"):
        assert torch.equal(a[k], b[k])
