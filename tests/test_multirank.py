"""Multi-rank host paths with two ranks on CPU (gloo).

Two splits, both without any data-path exchange:
  * independent problems (the bench's weak-scaling mode): each rank runs its own
    problem of the workload's shape; the only collectives are the two
    reductions of the timing result (max of the timed-region duration, sum of
    the executed FLOPs);
  * head sharding of one problem (``sharding``): each rank computes the heads
    it owns and one all_gather assembles O.  Here the oracle stands in for each
    rank's compute, and the assembled O must equal the single-rank result bit
    for bit.
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

        # head sharding of one problem (the tiny workload with 3 heads: shares 2 and 1)
        import oracle as Or
        from block_sparse_linear_pool_b200 import sharding as S
        one, w = I.make_workload("tiny_sla", H=3)
        f64 = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
        p = Or.OracleParams(k_h=w["k_h"], k_l=w["k_l"], combine="proj")
        Qs, Ks, Vs = (f64(S.head_slice(one[k], 3, rank, world)) for k in ("Q", "K", "V"))
        o_local, _ = Or.forward(Qs, Ks, Vs, p, proj_w=f64(one["proj_w"]))
        O_all = S.gather_heads(torch.from_numpy(o_local), 3)
        out[("sharded", rank)] = (O_all.numpy(), S.head_range(3, rank, world))
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


def test_head_sharded_forward_equals_the_single_rank_result(two_ranks):
    import oracle as Or
    from block_sparse_linear_pool_b200 import inputs as I

    one, w = I.make_workload("tiny_sla", H=3)
    f64 = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
    p = Or.OracleParams(k_h=w["k_h"], k_l=w["k_l"], combine="proj")
    ref, _ = Or.forward(f64(one["Q"]), f64(one["K"]), f64(one["V"]), p, proj_w=f64(one["proj_w"]))
    assert [two_ranks[("sharded", r)][1] for r in range(2)] == [(0, 2), (2, 3)]
    for r in range(2):
        np.testing.assert_array_equal(two_ranks[("sharded", r)][0], ref)


def test_head_ranges_cover_every_head_once():
    from block_sparse_linear_pool_b200 import sharding as S

    for H in (1, 2, 3, 12, 40):
        for world in (1, 2, 3, 8):
            rs = [S.head_range(H, r, world) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
            sizes = [b - a for a, b in rs]
            assert max(sizes) - min(sizes) <= 1


def test_problem_zero_is_the_default_instance():
    from block_sparse_linear_pool_b200 import inputs as I

    a, _ = I.make_workload("tiny_sla")
    b, _ = I.make_workload("tiny_sla", problem=0)
    for k in ("Q", "K", "V"):
        assert torch.equal(a[k], b[k])
