"""The N > 1 host path of bench.py on CPU: two gloo ranks reduce their step
times to the max over ranks and report all ranks' tokens over that time (every
rank runs an independent replica; the forward itself has no collective)."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + 5.0 * rank, 20.0 - 3.0 * rank]      # rank 1 is slower on the first timing
        got = bench.reduce_max(mine, "cpu")
        out[rank] = got
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_max_reduction_and_job_value():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
    assert out[0] == out[1] == [15.0, 20.0]
    # 2 replicas x (B=2, L=32760 tokens) over the slowest rank's 500 ms
    assert bench.whole_job_tokens_per_s(2, 2, 32760, 500.0) == pytest.approx(4 * 32760 / 0.5)


def test_single_process_reduce_is_identity():
    assert bench.reduce_max([3.0, 4.0], "cpu") == [3.0, 4.0]
