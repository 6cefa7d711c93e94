"""The multi-GPU path is independent replicas (no data-path collective):
world-size-2 gloo ranks on the CPU check the rank plumbing of bench.py --
independent seeds, max-over-ranks timing, whole-job weak-scaling value."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        w, r, lr = bench.rank_env()
        ms = 10.0 + 5.0 * r  # rank 1 is the slow one
        out[r] = (w, r, lr, bench.rank_seed(r), bench.max_over_ranks(ms, dist, "cpu"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert set(res) == {0, 1}
    for r in (0, 1):
        w, rr, lr, seed, mx = res[r]
        assert (w, rr, lr) == (2, r, r)
        assert mx == 15.0  # every rank sees the slowest rank's time
    assert res[0][3] != res[1][3]  # independent batches


def test_weak_scaling_value_and_single_rank():
    # units of all ranks over the slowest time, in giga-units per second
    assert bench.weak_scaling_value(4, 25_165_824, 100, 30.0) == pytest.approx(
        4 * 25_165_824 * 100 / 0.03 / 1e9)
    assert bench.max_over_ranks(7.5, None) == 7.5
