"""The multi-rank host logic of bench.py, run as two gloo ranks on the CPU: every rank draws its own
units (distinct seeds), the timed region is the max over ranks, and the whole-job value is weak
scaling (per-GPU work fixed).  No GPU and no data-path collective are involved."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys

    import torch.distributed as dist

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    w, r, lr = bench.rank_env()
    slowest = bench.max_over_ranks(10.0 + 5.0 * r, dist)  # rank-dependent "elapsed ms"
    out[rank] = (w, r, lr, bench.rank_seed(r), slowest)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_time_as_the_slowest_and_scale_weakly():
    import bench

    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    assert all(v[0] == world and v[1] == k and v[2] == k for k, v in res.items())
    assert res[0][3] != res[1][3]                # independent units per rank
    assert res[0][4] == res[1][4] == 15.0        # both ranks report the slowest rank's time
    one = bench.weak_scaling_value(1, 1e9, 10, 100.0)
    two = bench.weak_scaling_value(2, 1e9, 10, 100.0)
    assert two == pytest.approx(2 * one)         # same per-rank work and time: twice the job throughput
