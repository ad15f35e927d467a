"""The multi-rank plumbing of bench.py on CPU: two gloo ranks (one process
each, as torchrun launches them) agree on the slowest rank's time, and the
whole-job throughput counts every rank's tokens over that time."""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import bench
    w, r, _ = bench.dist_setup(backend="gloo")
    try:
        torch.distributed.barrier()
        my_ms = 10.0 + 5.0 * r  # rank 1 is the slow one
        m = bench.ranks_max(my_ms, w, "cpu")
        out[r] = (w, r, m, bench.job_tokens_per_s(1, 200, w, m))
        torch.distributed.barrier()
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world = 2
    with mp.get_context("spawn").Manager() as man:
        out = man.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    for r in range(world):
        w, rr, m, tps = res[r]
        assert (w, rr) == (world, r)
        assert m == 15.0                      # max over ranks, identical on every rank
        assert tps == pytest.approx(1 * 200 * 2 / 15e-3)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.ranks_max(3.5, 1, "cpu") == 3.5
    assert bench.job_tokens_per_s(4096, 10, 1, 100.0) == pytest.approx(409600.0)
