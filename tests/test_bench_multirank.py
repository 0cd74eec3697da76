"""CPU, two gloo ranks: the replica path of bench.py (one independent stream
per GPU, no collective on the data path) takes the slowest rank's time and
reports the whole job's throughput."""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank 1 is the slow replica
        times = [1.0 + rank, 2.0 * (rank + 1), 0.5, 3.0 - rank]
        got = bench.max_over_ranks(times, world, "cpu")
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0] == out[1] == [2.0, 4.0, 0.5, 3.0]


def test_job_throughput_counts_every_replica():
    one = bench.job_throughput(1e12, 1.0, 1)
    assert one == pytest.approx(1000.0)
    assert bench.job_throughput(1e12, 1.0, 8) == pytest.approx(8 * one)
    # slower step, lower throughput
    assert bench.job_throughput(1e12, 2.0, 2) == pytest.approx(one)


def test_attention_flops_of_the_headline_workload():
    w = bench.workload()
    # 4680 queries x 34,320 cached keys + 1560 x (1560 + 3120 + 4680) chunk pairs, per head
    assert bench.visible_pairs_per_head(w) == 4680 * 34320 + 1560 * 9360
    assert bench.attn_flops(w) == pytest.approx(1.0765467648e12, rel=1e-9)
