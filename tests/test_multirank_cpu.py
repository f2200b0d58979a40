"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The hot path has no exchange step; N GPUs run replicas, and the only
cross-rank steps are a barrier and the max-over-ranks of the device time.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        dist.barrier()
        m = bench.max_over_ranks(times[rank], dist, "cpu")
        v = bench.job_throughput(world, 1000, 10, m)
        out[rank] = (m, v)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_throughput_world_2():
    world = 2
    times = [12.5, 17.25]  # ms of device time per rank
    mgr = mp.get_context("spawn").Manager()  # no fork of a threaded process
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), times, out), nprocs=world, join=True)
    for rank in range(world):
        m, v = out[rank]
        assert m == pytest.approx(17.25)
        assert v == pytest.approx(world * 1000 * 10 / 0.01725)


def test_single_rank_helpers():
    assert bench.max_over_ranks(3.0) == 3.0
    assert bench.job_throughput(1, 65520, 30, 1000.0) == pytest.approx(65520 * 30)


def test_algorithmic_work_counts():
    """Pair count of the bench workload: per (b,h), chunk t has
    (end - first)*HW queries and (end - w)*HW window keys."""
    w = bench.algorithmic_work(2, 12, 21, 1560, 128, 128, 3, 1, False)
    pairs = 4680 * 4680 + 6 * (4680 * 6240)
    assert w["exps"] == pytest.approx(24 * pairs)
    assert w["attn_flops"] == pytest.approx(24 * (4 * 128 * pairs + 2 * 32760 * 128 * 128
                                                  + 2 * 32760 * 128 * 128 + 2 * 32760 * 128))
    assert w["full_softmax_flops"] / w["total_flops"] > 5.0
