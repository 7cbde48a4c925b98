"""The bench's multi-GPU bookkeeping on CPU: world_size 2 over gloo.  bench.py at N > 1 runs one
independent replica of the stack per GPU (the decode-step GEMV path has no cross-GPU exchange);
what it must get right is the max over ranks of the timed region and the whole-job throughput."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [2.0, 3.5][rank]  # rank 1 is the slower replica
        m = bench.max_over_ranks(ms, world, device="cpu")
        other = bench.max_over_ranks([7.0, 1.0][rank], world, device="cpu")  # every rank, same order
        out[rank] = (m, other, bench.whole_job_gbs(1e9, world, m))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_throughput_gloo():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
    for rank in range(world):
        m, other, gbs = out[rank]
        assert m == 3.5 and other == 7.0
        assert gbs == pytest.approx(2 * 1e9 / 3.5e-3 / 1e9)


def test_single_rank_passthrough():
    assert bench.max_over_ranks(1.25, 1, device="cpu") == 1.25
    assert bench.whole_job_gbs(2e9, 1, 0.5) == pytest.approx(4000.0)
