"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

Each rank runs its own batch (weak scaling, no data-path collective); the only
collectives are the barrier and the max over ranks of the timed span.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import torch

    import bench

    w, r, lr = bench.dist_env()
    dist = bench.init_dist(w, "gloo")
    dev = torch.device("cpu")
    bench.barrier(dist, dev)
    slowest = bench.max_over_ranks(10.0 * (rank + 1), dist, dev)  # rank 1 took 20 ms
    value = bench.weak_scaling_value(32768, w, slowest / 1e3)
    q.put((rank, w, slowest, value))
    dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_sum_the_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, world, slowest, value in out:
        assert world == 2
        assert slowest == 20.0
        assert value == pytest.approx(2 * 32768 / 0.020)


def test_single_rank_needs_no_process_group():
    import bench

    assert bench.init_dist(1, "gloo") is None
    assert bench.max_over_ranks(3.5, None, None) == 3.5
    assert bench.weak_scaling_value(100, 1, 0.5) == 200.0
