"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the timing is the max over ranks,
the throughput counts every rank's tokens, and each rank draws its own batch."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    import workloads as W
    ms = bench.max_over_ranks(10.0 + 5.0 * rank)
    cfg = W.scaled_config("switch", m=64, d=32, d_ff=64, seg_len=64, capacity=2)
    x = W.make_router_inputs(cfg, seed=bench.rank_seed(rank))["x"]
    out[rank] = (ms, float(x[0, 0]))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_throughput_gloo():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    assert out[0][0] == out[1][0] == 15.0  # every rank sees the slowest rank's time
    assert out[0][1] != out[1][1]          # ranks draw different batches
    import bench
    assert bench.whole_job_tokens_per_s(8192, 10, 2, 15.0) == pytest.approx(8192 * 10 * 2 / 0.015)
    assert bench.max_over_ranks(3.5) == 3.5  # no process group: identity
