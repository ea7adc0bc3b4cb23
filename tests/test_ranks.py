"""The multi-rank side of bench.py on CPU (gloo, world size 2): the layer
does not shard (each rank runs an independent replica), so the only
cross-rank step is the timing reduction -- every rank gets the max over
ranks, and the job rate counts every rank's tokens over that time."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, values, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(values[rank], torch.device("cpu"))
        out[rank] = got
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    world, port = 2, _free_port()
    values = [3.25, 7.5]
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_rank_main, args=(world, port, values, out), nprocs=world, start_method="spawn", join=True)
    assert out[0] == out[1] == max(values)


def test_single_process_keeps_its_value():
    assert bench.max_over_ranks(4.5, torch.device("cpu")) == 4.5


@pytest.mark.parametrize("world", [1, 2, 8])
def test_job_rate_counts_every_rank(world):
    # 8192 tokens per rank in 10 ms (the slowest rank) -> world * 819200 tokens/s
    assert bench.job_rate(8192, 10.0, world) == pytest.approx(world * 819200.0)
