"""Host logic of `bench.py --gpus N` (replicas, weak scaling) on CPU: two
`gloo` ranks, each timing its own replica, agree on the slowest rank's time,
draw different token streams and report the whole job's tokens over it.
"""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mine = 10.0 + 5.0 * rank                      # this replica's timed ms
        slowest = bench.max_over_ranks(mine, dist, torch.device("cpu"))
        seeds = [bench.step_seed(i, rank) for i in range(3)]
        out[rank] = (mine, slowest, seeds, bench.job_tokens_per_s(world, 4, 8, slowest))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_max_time_and_distinct_streams():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    assert sorted(out.keys()) == [0, 1]
    slowest = {out[r][1] for r in range(world)}
    assert slowest == {15.0}                               # every rank holds the max over ranks
    assert not set(out[0][2]) & set(out[1][2])             # replicas draw disjoint token streams
    # whole job: 2 replicas x 4 steps x 8 tokens over the slowest rank's 15 ms
    assert out[0][3] == pytest.approx(2 * 4 * 8 / 15e-3)


def test_single_process_paths():
    import bench
    assert bench.max_over_ranks(3.5, None, None) == 3.5
    assert bench.job_tokens_per_s(1, 10, 1, 1.0) == pytest.approx(10000.0)
    assert bench.step_seed(0, 0) == bench.X_SEED0
